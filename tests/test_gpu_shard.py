"""The shard entry points on one GPU: two "ranks" with caches of their own blocks only.

The context's blocks are split into two ranges (``block_range``).  Each emulated rank has
its own paged cache whose page table maps only the logical pages it may read (its blocks,
the anchor block's pages for a rank after the first, and the tail on the rank with the last
block) and points every other logical page past the pools: a read outside the rank's range
would be clamped and reported by star_device_status, so the test also shows that no kernel
strays.  The ranks run Phase 1 on their blocks (star_phase1_encode_shard), their Phase-2
partials (star_phase2_partial_shard) and every decode step's partial
(star_decode_partial_shard); the partials are concatenated, as the all-gather of the
multi-GPU exchange lays them out, and merged by star_lse_merge.  Results are compared with
the oracle, and the Phase-1 rows bit for bit with the unsharded call.
"""

import numpy as np
import pytest
import torch

import oracle
from synth import Workload, make_inputs

pytestmark = pytest.mark.gpu

CASES = {
    "d128-g4-n4": Workload("shard-d128-g4-n4", B=2, Hq=8, Hkv=2, d=128, L=2048, b=512, T=40, S=3, peaky=True),
    "d64-g2-n5-a256": Workload("shard-d64-g2-n5", B=1, Hq=4, Hkv=2, d=64, L=1280, b=256, T=7, S=2, peaky=False,
                               anchor=128),
}


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _rank_cache(star, shape, wl, i0, i1):
    """A cache whose page table maps only what blocks [i0, i1) may read."""
    max_pages = star.star_pages_needed(shape)
    P = wl.page_tokens
    readable = set(range(i0 * wl.b // P, i1 * wl.b // P))
    if i0 > 0:
        readable |= set(range(0, -(-wl.a // P)))          # the anchor's pages
    if i1 == wl.n:
        readable |= set(range(wl.L // P, max_pages))       # the tail
    num_pages = wl.B * len(readable)
    pt = torch.full((wl.B, max_pages), num_pages + 3, dtype=torch.int32)  # past the pools
    nxt = 0
    for bi in range(wl.B):
        for j in sorted(readable):
            pt[bi, j] = nxt
            nxt += 1
    return star.PagedKVCache(shape, page_table=pt, num_pages=num_pages)


@pytest.mark.parametrize("name", list(CASES))
def test_two_shards_match_the_oracle_and_the_unsharded_phase1(name):
    import block_sparse_attention_star_b200 as star
    from block_sparse_attention_star_b200.shard import block_range
    from tests import harness as h
    wl = CASES[name]
    inp = make_inputs(wl, "cuda")
    shape = h.shape_of(wl)
    ref = oracle.run_star(h.oracle_inputs(inp), wl.L, wl.b, wl.theta, anchor=wl.anchor or None)
    full = h.run_gpu(wl, inp, phases=("phase1",))
    ranges = [block_range(wl.n, 2, r) for r in range(2)]
    T, S, a = wl.T, wl.S, wl.a
    caches = [_rank_cache(star, shape, wl, i0, i1) for i0, i1 in ranges]
    # Phase 1 per rank: its rows, bit-identical to the unsharded call.
    for (i0, i1), cache in zip(ranges, caches):
        sl = slice(i0 * wl.b, i1 * wl.b)
        q, k, v = (inp[x][:, sl].contiguous() for x in ("q_ctx", "k_ctx", "v_ctx"))
        pos = inp["pos_ctx"][:, sl].contiguous()
        ka, va = inp["k_ctx"][:, :a].contiguous(), inp["v_ctx"][:, :a].contiguous()
        pa = inp["pos_ctx"][:, :a].contiguous()
        out = torch.empty_like(q)
        star.star_phase1_encode_shard(shape, cache, star.StarShard(i0, i1), q, k, v, pos, ka, va, pa, out)
        torch.cuda.synchronize()
        assert star.star_device_status() == 0
        assert torch.equal(out, full["o_ctx"][:, sl]), f"rank blocks [{i0}, {i1}): Phase-1 rows differ"
        h.assert_out(out, ref["o_ctx"][:, sl], f"phase1 shard [{i0}, {i1})")
    # Phase 2: each rank's partials (only the last rank appends the query's K/V), in block order.
    rows = wl.B * T * wl.Hq
    o_parts, l_parts = [], []
    for (i0, i1), cache in zip(ranges, caches):
        o = torch.empty((i1 - i0, wl.B, T, wl.Hq, wl.d), dtype=torch.float32, device="cuda")
        l = torch.empty((i1 - i0, wl.B, T, wl.Hq), dtype=torch.float32, device="cuda")
        ws = star.workspace(shape, star.STAR_OP_PHASE2, T)
        tail = i1 == wl.n
        star.star_phase2_partial_shard(shape, cache, star.StarShard(i0, i1), inp["q_query"],
                                       inp["k_query"] if tail else None, inp["v_query"] if tail else None,
                                       inp["pos_query"], T, o, l, ws)
        o_parts.append(o)
        l_parts.append(l)
    o_all, l_all = torch.cat(o_parts), torch.cat(l_parts)
    torch.cuda.synchronize()
    assert star.star_device_status() == 0
    h.assert_out(o_all, ref["o_part"], "phase2 shard partials O")
    h.assert_lse(l_all, ref["lse_part"], "phase2 shard partials LSE")
    o_q = torch.empty((wl.B, T, wl.Hq, wl.d), dtype=torch.bfloat16, device="cuda")
    l_q = torch.empty((wl.B, T, wl.Hq), dtype=torch.float32, device="cuda")
    star.star_lse_merge(wl.n, rows, wl.d, o_all, l_all, o_q, l_q)
    h.assert_out(o_q, ref["o_query"], "sharded query output")
    h.assert_lse(l_q, ref["lse_query"], "sharded query LSE")
    # Decode: every step, one partial per rank (the last rank appends the token), merged.
    wsd = [star.workspace(shape, star.STAR_OP_DECODE) for _ in ranges]
    for s in range(S):
        po = torch.empty((2, wl.B, wl.Hq, wl.d), dtype=torch.float32, device="cuda")
        pl = torch.empty((2, wl.B, wl.Hq), dtype=torch.float32, device="cuda")
        for r, ((i0, i1), cache) in enumerate(zip(ranges, caches)):
            star.star_decode_partial_shard(shape, cache, star.StarShard(i0, i1), inp["q_dec"][s], inp["k_dec"][s],
                                           inp["v_dec"][s], inp["pos_dec"][s], wl.L + T + s, po[r], pl[r], wsd[r])
        o_d = torch.empty((wl.B, wl.Hq, wl.d), dtype=torch.bfloat16, device="cuda")
        l_d = torch.empty((wl.B, wl.Hq), dtype=torch.float32, device="cuda")
        star.star_lse_merge(2, wl.B * wl.Hq, wl.d, po, pl, o_d, l_d)
        torch.cuda.synchronize()
        h.assert_out(o_d, ref["o_dec"][s], f"sharded decode step {s} O")
        h.assert_lse(l_d, ref["lse_dec"][s], f"sharded decode step {s} LSE")
    assert star.star_device_status() == 0


def test_shard_arguments_are_checked_before_any_launch():
    import block_sparse_attention_star_b200 as star
    from tests import harness as h
    wl = CASES["d128-g4-n4"]
    shape = h.shape_of(wl)
    cache = star.PagedKVCache(shape)
    inp = make_inputs(wl, "cuda", parts=("query",))
    o = torch.empty((2, wl.B, wl.T, wl.Hq, wl.d), dtype=torch.float32, device="cuda")
    l = torch.empty((2, wl.B, wl.T, wl.Hq), dtype=torch.float32, device="cuda")
    ws = star.workspace(shape, star.STAR_OP_PHASE2, wl.T)
    for bad in ((2, 2), (3, 5), (-1, 1)):
        with pytest.raises(star.StarError) as e:
            star.star_phase2_partial_shard(shape, cache, star.StarShard(*bad), inp["q_query"], None, None,
                                           inp["pos_query"], wl.T, o, l, ws)
        assert e.value.code == star.STAR_ERR_INVALID_ARG
    # k, v off the last block: only the tail's owner appends.
    with pytest.raises(star.StarError) as e:
        star.star_phase2_partial_shard(shape, cache, star.StarShard(0, 2), inp["q_query"], inp["k_query"],
                                       inp["v_query"], inp["pos_query"], wl.T, o, l, ws)
    assert e.value.code == star.STAR_ERR_INVALID_ARG
    assert star.star_device_status() == 0
