"""The exchange over peer memory on one GPU.

star_phase2_partial_shard_push / star_decode_partial_shard_push store a shard's partials into
slot `rank` of every rank's exchange buffer; star_exchange_merge waits for all ranks' slots of
an epoch in its own buffer and merges them.  On one GPU the ranks are emulated in one process:
their buffers are ordinary device buffers, every rank's view lists all of them, and the calls
run in stream order (every rank pushes an epoch before any rank merges it), so no wait depends
on a kernel that has not been launched.  Results are compared with the oracle and with the
collective-free path (star_phase2_partial_shard + star_lse_merge).  A merge whose partials never
arrive shows that the wait is bounded: STAR_ERR_TIMEOUT, and the context stays usable.
"""

import ctypes

import pytest
import torch

import oracle
from synth import Workload, make_inputs
from tests.test_gpu_shard import _rank_cache

pytestmark = pytest.mark.gpu

WL = Workload("xchg-d128-g4-n4", B=2, Hq=8, Hkv=2, d=128, L=2048, b=512, T=40, S=4, peaky=True)


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _buffers(star, world, slots, rows, d):
    size = star.star_exchange_size(world, slots, rows, d)
    bufs = [torch.zeros(size, dtype=torch.uint8, device="cuda") for _ in range(world)]
    views = [star.StarExchange(world, r, slots, (ctypes.c_void_p * 8)(*[b.data_ptr() for b in bufs]))
             for r in range(world)]
    return bufs, views


@pytest.mark.parametrize("world", [1, 2, 3])
def test_peer_exchange_matches_the_oracle(world):
    """world 3 splits the 4 blocks 2 + 1 + 1: the ranks with one block pad their second slot
    with an empty partial."""
    import block_sparse_attention_star_b200 as star
    from block_sparse_attention_star_b200.shard import block_range
    from tests import harness as h
    wl = WL
    inp = make_inputs(wl, "cuda")
    shape = h.shape_of(wl)
    ref = oracle.run_star(h.oracle_inputs(inp), wl.L, wl.b, wl.theta)
    ranges = [block_range(wl.n, world, r) for r in range(world)]
    slots = max(e - b for b, e in ranges)
    T, S = wl.T, wl.S
    caches = []
    for (i0, i1) in ranges:
        cache = _rank_cache(star, shape, wl, i0, i1)
        sl = slice(i0 * wl.b, i1 * wl.b)
        q, k, v = (inp[x][:, sl].contiguous() for x in ("q_ctx", "k_ctx", "v_ctx"))
        out = torch.empty_like(q)
        star.star_phase1_encode_shard(shape, cache, star.StarShard(i0, i1), q, k, v, inp["pos_ctx"][:, sl].contiguous(),
                                      inp["k_ctx"][:, :wl.a].contiguous(), inp["v_ctx"][:, :wl.a].contiguous(),
                                      inp["pos_ctx"][:, :wl.a].contiguous(), out)
        caches.append(cache)
    # Phase 2: every rank pushes epoch 1, then every rank merges it.
    rows = wl.B * T * wl.Hq
    _, xq = _buffers(star, world, slots, rows, wl.d)
    ws = [star.workspace(shape, star.STAR_OP_PHASE2_PUSH, T) for _ in ranges]
    for r, (i0, i1) in enumerate(ranges):
        tail = i1 == wl.n
        star.star_phase2_partial_shard_push(shape, caches[r], star.StarShard(i0, i1), inp["q_query"],
                                            inp["k_query"] if tail else None, inp["v_query"] if tail else None,
                                            inp["pos_query"], T, xq[r], 1, ws[r])
    outs = []
    for r in range(world):
        o = torch.empty((wl.B, T, wl.Hq, wl.d), dtype=torch.bfloat16, device="cuda")
        l = torch.empty((wl.B, T, wl.Hq), dtype=torch.float32, device="cuda")
        star.star_exchange_merge(xq[r], rows, wl.d, 1, o, l)
        outs.append((o, l))
    torch.cuda.synchronize()
    assert star.star_device_status() == 0
    for o, l in outs:
        h.assert_out(o, ref["o_query"], f"exchanged query output (world {world})")
        h.assert_lse(l, ref["lse_query"], f"exchanged query LSE (world {world})")
        assert torch.equal(o, outs[0][0]) and torch.equal(l, outs[0][1]), "ranks disagree"
    # Decode: one exchange per step (epochs 1..S on a buffer of one slot; parities reused).
    drows = wl.B * wl.Hq
    _, xd = _buffers(star, world, 1, drows, wl.d)
    wsd = [star.workspace(shape, star.STAR_OP_DECODE) for _ in ranges]
    for s in range(S):
        for r, (i0, i1) in enumerate(ranges):
            star.star_decode_partial_shard_push(shape, caches[r], star.StarShard(i0, i1), inp["q_dec"][s],
                                                inp["k_dec"][s], inp["v_dec"][s], inp["pos_dec"][s], wl.L + T + s,
                                                xd[r], s + 1, wsd[r])
        for r in range(world):
            o = torch.empty((wl.B, wl.Hq, wl.d), dtype=torch.bfloat16, device="cuda")
            l = torch.empty((wl.B, wl.Hq), dtype=torch.float32, device="cuda")
            star.star_exchange_merge(xd[r], drows, wl.d, s + 1, o, l)
            torch.cuda.synchronize()
            h.assert_out(o, ref["o_dec"][s], f"exchanged decode step {s} (rank {r} of {world})")
            h.assert_lse(l, ref["lse_dec"][s], f"exchanged decode step {s} LSE (rank {r} of {world})")
    assert star.star_device_status() == 0


def test_exchange_merge_with_nothing_pushed_times_out_and_the_context_stays_usable():
    import block_sparse_attention_star_b200 as star
    import time
    _, x = _buffers(star, 2, 1, 32, 128)
    o = torch.empty((32, 128), dtype=torch.bfloat16, device="cuda")
    star.star_debug_set(20_000_000, 0)
    try:
        t0 = time.monotonic()
        star.star_exchange_merge(x[0], 32, 128, 3, o)   # rank 1 never pushes epoch 3
        torch.cuda.synchronize()
        elapsed = time.monotonic() - t0
    finally:
        star.star_debug_set(0, 0)
    with pytest.raises(star.StarError) as e:
        star.star_device_status()
    assert e.value.code == star.STAR_ERR_TIMEOUT
    assert elapsed < 5.0
    assert star.star_device_status() == 0


def test_exchange_arguments_are_checked():
    import block_sparse_attention_star_b200 as star
    _, x = _buffers(star, 2, 1, 32, 128)
    o = torch.empty((32, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(star.StarError) as e:
        star.star_exchange_merge(x[0], 32, 128, 0, o)             # epochs start at 1
    assert e.value.code == star.STAR_ERR_INVALID_ARG
    bad = star.StarExchange(9, 0, 1, (ctypes.c_void_p * 8)(*[x[0].peers[0]] * 8))
    with pytest.raises(star.StarError) as e:
        star.star_exchange_merge(bad, 32, 128, 1, o)
    assert e.value.code == star.STAR_ERR_UNSUPPORTED_SHAPE
    assert star.star_device_status() == 0
