"""Failure detection on the GPU, without faulting or hanging it.

Every mbarrier wait in the attention and decode kernels is bounded: when it runs
out, the kernel records an error code in a device word and returns, and
star_device_status reports STAR_ERR_TIMEOUT.  These tests make the waits run out
on purpose through the library's test hook (star_debug_set): CTA 0's producer
issues no first K-tile load, so the barrier of that stage never completes -- a
flag that nothing sets -- and nothing asynchronous is left in flight.  The wait
limit is shortened to 20 ms for the test.  Afterwards the hook is switched off and
the same calls must give results bit-identical to a clean run, showing that the
context stayed usable.

A page-table entry outside [0, num_pages) is clamped by the kernels (no access
leaves the pools) and reported as STAR_ERR_CAPACITY.
"""

import time

import pytest
import torch

from synth import Workload, make_inputs

pytestmark = pytest.mark.gpu

WL = Workload("fail-d128", B=1, Hq=8, Hkv=2, d=128, L=2048, b=512, T=40, S=2, peaky=False)


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    import block_sparse_attention_star_b200 as star
    star.star_debug_set(0, 0)


def _expect_timeout(star, what):
    with pytest.raises(star.StarError) as e:
        star.star_device_status()
    assert e.value.code == star.STAR_ERR_TIMEOUT, f"{what}: {e.value}"
    assert star.star_device_status() == 0, f"{what}: the error word was not cleared"


@pytest.mark.parametrize("step", ["phase1", "phase2", "decode"])
def test_bounded_waits_give_up_and_the_context_stays_usable(step):
    import block_sparse_attention_star_b200 as star
    from tests import harness
    inp = make_inputs(WL, "cuda")
    clean = harness.run_gpu(WL, inp)
    assert clean["status"] == 0
    shape, cache = clean["shape"], clean["cache"]
    star.star_debug_set(20_000_000, star.STAR_DEBUG_SKIP_FIRST_LOAD)
    try:
        torch.cuda.synchronize()
        t0 = time.monotonic()
        if step == "phase1":
            out = torch.empty_like(inp["q_ctx"])
            star.star_phase1_encode(shape, cache, inp["q_ctx"], inp["k_ctx"], inp["v_ctx"], inp["pos_ctx"], out)
        elif step == "phase2":
            o_part, lse_part = star.alloc_partials(shape, WL.T)
            ws = star.workspace(shape, star.STAR_OP_PHASE2, WL.T)
            star.star_phase2_partial(shape, cache, inp["q_query"], None, None, inp["pos_query"], WL.T, o_part,
                                     lse_part, ws)
        else:
            o = torch.empty((WL.B, 1, WL.Hq, WL.d), dtype=torch.bfloat16, device="cuda")
            lse = torch.empty((WL.B, WL.Hq), dtype=torch.float32, device="cuda")
            wsd = star.workspace(shape, star.STAR_OP_DECODE)
            # the clean run's last decode step again (same token, same slot)
            s = WL.S - 1
            star.star_decode_step(shape, cache, inp["q_dec"][s], inp["k_dec"][s], inp["v_dec"][s],
                                  inp["pos_dec"][s], WL.L + WL.T + s, o, lse, wsd)
        torch.cuda.synchronize()
        elapsed = time.monotonic() - t0
    finally:
        star.star_debug_set(0, 0)
    _expect_timeout(star, step)
    assert elapsed < 5.0, f"{step}: the bounded waits took {elapsed:.2f} s with a 20 ms limit"
    again = harness.run_gpu(WL, inp)
    assert again["status"] == 0
    for key in ("o_ctx", "o_part", "lse_part", "o_query", "lse_query", "o_dec", "lse_dec"):
        assert torch.equal(clean[key], again[key]), f"after the {step} timeout: {key} differs from the clean run"


def test_out_of_range_page_entry_is_reported_and_clamped():
    import block_sparse_attention_star_b200 as star
    from tests import harness
    inp = make_inputs(WL, "cuda")
    shape = harness.shape_of(WL)
    good = star.PagedKVCache(shape)
    pt = good.page_table.clone()
    pt[0, 3] = good.num_pages + 5                      # logical page 3 points past the pools
    bad = star.PagedKVCache(shape, page_table=pt.cpu(), num_pages=good.num_pages)
    out = torch.empty_like(inp["q_ctx"])
    star.star_phase1_encode(shape, bad, inp["q_ctx"], inp["k_ctx"], inp["v_ctx"], inp["pos_ctx"], out)
    with pytest.raises(star.StarError) as e:
        star.star_device_status()
    assert e.value.code == star.STAR_ERR_CAPACITY and "page-table entry" in str(e.value)
    # The next call with a valid table is clean.
    star.star_phase1_encode(shape, good, inp["q_ctx"], inp["k_ctx"], inp["v_ctx"], inp["pos_ctx"], out)
    assert star.star_device_status() == 0
