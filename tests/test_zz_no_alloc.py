"""The allocation-free decode entry point agrees with the workspace one.

star_decode_step_noalloc is for callers that cannot call cudaMalloc (a runtime
whose device memory is all reserved up front, a plugin handed only its input and
output buffers).  This file is collected last so that, if it fails, every other
test has already run.  It builds two identical caches, then decodes the same two
tokens in a row on each: through star_decode_step (caller workspace) and through
star_decode_step_noalloc (built-in scratch), called through the C ABI.  Both run
the same kernels on the same inputs, so the outputs must be bit-identical; they
are also checked against the CPU oracle.

The built-in scratch keeps whatever the previous call left in it.  Before the
compared calls, one no-alloc decode on a larger shape (more chunks, more rows)
fills it with other data, so a partial the kernel failed to write would be read
as that stale value and show up as a mismatch.
"""

import pytest
import torch

from synth import Workload, make_inputs

pytestmark = pytest.mark.gpu


def _prefill(wl, inp, star, harness):
    shape = harness.shape_of(wl)
    cache = star.PagedKVCache(shape)
    out = torch.empty_like(inp["q_ctx"])
    star.star_phase1_encode(shape, cache, inp["q_ctx"], inp["k_ctx"], inp["v_ctx"], inp["pos_ctx"], out)
    star.star_kv_append(shape, cache, inp["k_query"], inp["v_query"], inp["pos_query"], wl.L, wl.T)
    return shape, cache


def _poison_scratch(star, harness):
    """One no-alloc decode on a shape whose partials cover more of the scratch."""
    big = Workload("noalloc-poison", B=2, Hq=16, Hkv=2, d=128, L=16384, b=4096, T=16, S=1, peaky=False, seed=7)
    inp = make_inputs(big, "cuda")
    shape, cache = _prefill(big, inp, star, harness)
    o = torch.empty((big.B, 1, big.Hq, big.d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((big.B, big.Hq), dtype=torch.float32, device="cuda")
    star.star_decode_step_noalloc(shape, cache, inp["q_dec"][0], inp["k_dec"][0], inp["v_dec"][0], inp["pos_dec"][0],
                                  big.L + big.T, o, lse)
    torch.cuda.synchronize()
    assert torch.isfinite(lse).all()


@pytest.mark.parametrize("wl", [
    Workload("noalloc-d128", B=2, Hq=8, Hkv=2, d=128, L=2048, b=512, T=40, S=2, peaky=True),
    Workload("noalloc-d64", B=1, Hq=4, Hkv=1, d=64, L=1024, b=256, T=16, S=2, peaky=False),
])
def test_noalloc_decode_matches_workspace_decode(wl):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import block_sparse_attention_star_b200 as star
    import oracle
    from tests import harness
    _poison_scratch(star, harness)
    inp = make_inputs(wl, "cuda")
    shape_a, cache_a = _prefill(wl, inp, star, harness)
    shape_b, cache_b = _prefill(wl, inp, star, harness)
    ws = star.workspace(shape_a, star.STAR_OP_DECODE)
    ref = oracle.run_star(harness.oracle_inputs(inp), wl.L, wl.b, wl.theta, with_phase1=False)
    for s in range(2):
        cur = wl.L + wl.T + s
        ref_o = torch.empty((wl.B, 1, wl.Hq, wl.d), dtype=torch.bfloat16, device="cuda")
        ref_l = torch.empty((wl.B, wl.Hq), dtype=torch.float32, device="cuda")
        star.star_decode_step(shape_a, cache_a, inp["q_dec"][s], inp["k_dec"][s], inp["v_dec"][s], inp["pos_dec"][s],
                              cur, ref_o, ref_l, ws)
        got_o = torch.full_like(ref_o, float("nan"))
        got_l = torch.full_like(ref_l, float("nan"))
        star.star_decode_step_noalloc(shape_b, cache_b, inp["q_dec"][s], inp["k_dec"][s], inp["v_dec"][s],
                                      inp["pos_dec"][s], cur, got_o, got_l)
        torch.cuda.synchronize()
        assert torch.equal(got_o, ref_o), f"noalloc decode step {s}: O differs from the workspace decode"
        assert torch.equal(got_l, ref_l), f"noalloc decode step {s}: LSE differs from the workspace decode"
        harness.assert_out(got_o[:, 0], ref["o_dec"][s], f"noalloc decode step {s} O vs oracle")
        harness.assert_lse(got_l, ref["lse_dec"][s], f"noalloc decode step {s} LSE vs oracle")
    # Both caches received the same appended tokens.
    assert torch.equal(cache_a.k_pool, cache_b.k_pool) and torch.equal(cache_a.v_pool, cache_b.v_pool)
    assert star.star_device_status() == 0


def test_noalloc_rejects_shapes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import block_sparse_attention_star_b200 as star
    from tests import harness
    # 512 sequences x 64 query heads over a million-token cache: even one chunk per
    # (sequence, KV head) gives 32768 f32 output rows of 128 values, 16 MiB plus the
    # LSEs, more than the built-in scratch holds (rejected on the host, nothing runs).
    big = Workload("noalloc-big", B=512, Hq=64, Hkv=8, d=128, L=1 << 20, b=1 << 17, T=32, S=16, peaky=False)
    shape = harness.shape_of(big)
    assert star.star_workspace_size(shape, star.STAR_OP_DECODE) > 16 << 20
    small = Workload("noalloc-small", B=1, Hq=4, Hkv=1, d=64, L=1024, b=256, T=16, S=2, peaky=False)
    cache = star.PagedKVCache(harness.shape_of(small))
    q = torch.zeros((big.B, 1, big.Hq, big.d), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((big.B, 1, big.Hkv, big.d), dtype=torch.bfloat16, device="cuda")
    pos = torch.zeros(big.B, dtype=torch.int32, device="cuda")
    with pytest.raises(star.StarError) as e:
        star.star_decode_step_noalloc(shape, cache, q, kv, kv, pos, 0, q, None)
    assert e.value.code == star.STAR_ERR_CAPACITY and "16777216" in str(e.value)
