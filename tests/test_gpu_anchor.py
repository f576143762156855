"""GPU parity for the anchor variants: an anchor of the first a < b tokens of block 1,
and anchor position ids given per block ("Star Attention 完全拆解(一)", section
"仓库里的真实实现": anchor_block_size is a parameter of its own; the implementers'
notes there: the anchor's ids sampled from the prefix range, or reset to 0).

Full tensors at small shapes, sampled rows at the 8B 32K and 128K shapes, against
the oracle's literal c'; the same tolerances as the main parity tests.  An anchor of
the whole block given its own ids through the anchored call must reproduce
star_phase1_encode bit for bit (same keys, same kernel).
"""

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from synth import Workload, get_config, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def H():
    from tests import harness
    return harness


_tiny = get_config("tiny")
SMALL = {
    "tiny-a128-offset": dataclasses.replace(_tiny, name="tiny-a128-offset", anchor=128, anchor_ids="offset"),
    "tiny-a128-context": dataclasses.replace(_tiny, name="tiny-a128-context", anchor=128),
    "d128-g4-b2-zero": Workload("d128-g4-b2-zero", B=2, Hq=8, Hkv=2, d=128, L=2048, b=512, T=8, S=1, peaky=True,
                                anchor_ids="zero"),
    "d128-g8-a256-offset": Workload("d128-g8-a256-offset", B=1, Hq=16, Hkv=2, d=128, L=1536, b=512, T=8, S=1,
                                    peaky=True, anchor=256, anchor_ids="offset"),
}


def _oracle_phase1(wl, inp, bi):
    h = H()
    apos = inp["anchor_pos"][bi].cpu().numpy().astype(np.int64) if "anchor_pos" in inp else None
    O, _, _ = oracle.phase1(h.to64(inp["q_ctx"][bi]), h.to64(inp["k_ctx"][bi]), h.to64(inp["v_ctx"][bi]),
                            inp["pos_ctx"][bi].cpu().numpy().astype(np.int64), wl.b, wl.theta, wl.anchor or None, apos)
    return O


@pytest.mark.parametrize("name", list(SMALL))
def test_phase1_anchor_variants_match_oracle(name):
    wl = SMALL[name]
    h = H()
    inp = make_inputs(wl, "cuda")
    assert ("anchor_pos" in inp) == (wl.anchor_ids != "context")
    res = h.run_gpu(wl, inp, phases=("phase1",))
    assert res["status"] == 0
    for bi in range(wl.B):
        h.assert_out(res["o_ctx"][bi], _oracle_phase1(wl, inp, bi), f"{name} phase1 output (seq {bi})")


def test_anchor_with_its_own_ids_is_bit_identical_to_the_default():
    """a = b and ids 0..b-1 through the anchored call: the anchor's keys are roped into the
    workspace instead of read from the cache, and equal them bit for bit."""
    import block_sparse_attention_star_b200 as star
    h = H()
    wl = Workload("d128-ctx-ids", B=2, Hq=8, Hkv=2, d=128, L=1536, b=512, T=8, S=1, peaky=True)
    inp = make_inputs(wl, "cuda", parts=("ctx",))
    shape = h.shape_of(wl)
    apos = torch.arange(wl.b, dtype=torch.int32, device="cuda").repeat(wl.B, wl.n - 1, 1).contiguous()
    outs = []
    for anchored in (False, True):
        cache = star.PagedKVCache(shape)
        out = torch.empty_like(inp["q_ctx"])
        if anchored:
            ws = star.workspace(shape, star.STAR_OP_PHASE1_ANCHOR)
            star.star_phase1_encode_anchored(shape, cache, inp["q_ctx"], inp["k_ctx"], inp["v_ctx"], inp["pos_ctx"],
                                             apos, out, ws)
        else:
            star.star_phase1_encode(shape, cache, inp["q_ctx"], inp["k_ctx"], inp["v_ctx"], inp["pos_ctx"], out)
        torch.cuda.synchronize()
        assert star.star_device_status() == 0
        outs.append(out)
    assert torch.equal(outs[0], outs[1])


def test_anchored_call_rejects_a_small_workspace():
    import block_sparse_attention_star_b200 as star
    h = H()
    wl = SMALL["tiny-a128-offset"]
    inp = make_inputs(wl, "cuda", parts=("ctx",))
    shape = h.shape_of(wl)
    cache = star.PagedKVCache(shape)
    out = torch.empty_like(inp["q_ctx"])
    need = star.star_workspace_size(shape, star.STAR_OP_PHASE1_ANCHOR)
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(star.StarError) as e:
        star.star_phase1_encode_anchored(shape, cache, inp["q_ctx"], inp["k_ctx"], inp["v_ctx"], inp["pos_ctx"],
                                         inp["anchor_pos"], out, ws)
    assert e.value.code == star.STAR_ERR_CAPACITY


def test_build_positions_with_anchor_size_bit_exact():
    import block_sparse_attention_star_b200 as star
    h = H()
    wl = SMALL["d128-g8-a256-offset"]
    shape = h.shape_of(wl)
    cache = star.PagedKVCache(shape)
    pos = torch.arange(wl.L, dtype=torch.int32).repeat(wl.B, 1).cuda().contiguous()
    aug = torch.empty((wl.B, wl.L + (wl.n - 1) * wl.a), dtype=torch.int32, device="cuda")
    bmap = torch.empty((wl.B, wl.L, 3), dtype=torch.int32, device="cuda")
    star.star_build_positions(shape, cache, pos, aug, bmap)
    torch.cuda.synchronize()
    blocks = oracle.augmented_context(wl.L, wl.b, pos[0].cpu().numpy(), wl.a)
    assert np.array_equal(aug[0].cpu().numpy(), np.concatenate([blk["pos"] for blk in blocks]))


def _sampled(wl, rows_per_block):
    h = H()
    inp = make_inputs(wl, "cuda", parts=("ctx",))
    res = h.run_gpu(wl, inp, phases=("phase1",))
    assert res["status"] == 0
    rows = h.sample_rows(wl, rows_per_block)
    for bi in range(wl.B):
        apos = inp["anchor_pos"][bi].cpu().numpy().astype(np.int64) if "anchor_pos" in inp else None
        ref = oracle.phase1_rows(rows, h.to64(inp["q_ctx"][bi][torch.from_numpy(rows).cuda()]), h.to64(inp["k_ctx"][bi]),
                                 h.to64(inp["v_ctx"][bi]), inp["pos_ctx"][bi].cpu().numpy().astype(np.int64), wl.b,
                                 wl.theta, wl.anchor or None, apos)
        h.assert_out(res["o_ctx"][bi][torch.from_numpy(rows).cuda()], ref, f"{wl.name} sampled rows")


def test_llama8b_32k_quarter_anchor_offset_ids_sampled():
    wl = dataclasses.replace(get_config("llama8b-32k"), name="llama8b-32k-a2048-offset", anchor=2048,
                             anchor_ids="offset")
    _sampled(wl, 20)


@pytest.mark.parametrize("name", ["llama8b-128k-b32768-a8192-offset", "llama8b-128k-b32768-zero"])
def test_llama8b_128k_anchor_variants_sampled(name):
    _sampled(get_config(name), 6)
