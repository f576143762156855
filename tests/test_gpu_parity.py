"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Element-by-element at sizes the oracle finishes in seconds (several 128-row
tiles, ragged query tails, both head dims, GQA groups 2/4/8, one block, a
permuted page table); sampled rows plus full Phase-2/decode checks at the
Llama-3.1-8B 32K and 128K workloads.  Tolerances: max abs <= 1.5e-2 and mean
abs <= 2e-3 on outputs, abs <= 1e-3 on LSE; integer outputs bit-exact.
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


SMALL = {
    "tiny": get_config("tiny"),
    "d128-g4-b2": Workload("d128-g4-b2", B=2, Hq=8, Hkv=2, d=128, L=2048, b=512, T=40, S=5, peaky=True),
    "d128-n1": Workload("d128-n1", B=1, Hq=4, Hkv=2, d=128, L=512, b=512, T=20, S=3, peaky=False),
    "d128-g8-t130": Workload("d128-g8-t130", B=1, Hq=16, Hkv=2, d=128, L=1024, b=256, T=130, S=2, peaky=True),
    "d64-g2-p128": Workload("d64-g2-p128", B=1, Hq=4, Hkv=2, d=64, L=768, b=256, T=7, S=4, peaky=False,
                            page_tokens=128),
    # one query token; the decode slots and the query tail cross page boundaries (pages of 256)
    "d128-t1": Workload("d128-t1", B=1, Hq=8, Hkv=2, d=128, L=1024, b=256, T=1, S=3, peaky=True),
    "d128-pagecross": Workload("d128-pagecross", B=2, Hq=8, Hkv=2, d=128, L=1024, b=256, T=250, S=10,
                               peaky=False),
    "d64-g8": Workload("d64-g8", B=1, Hq=16, Hkv=2, d=64, L=1024, b=256, T=24, S=3, peaky=True),
    "d128-p512": Workload("d128-p512", B=1, Hq=8, Hkv=2, d=128, L=2048, b=512, T=16, S=3, peaky=False,
                          page_tokens=512),
}


def _full_compare(wl, page_table=None, num_pages=None):
    h = H()
    inp = make_inputs(wl, "cuda")
    res = h.run_gpu(wl, inp, page_table=page_table, num_pages=num_pages)
    assert res["status"] == 0
    ref = oracle.run_star(h.oracle_inputs(inp), wl.L, wl.b, wl.theta)
    h.assert_out(res["o_ctx"], ref["o_ctx"], "phase1 output")
    for bi in range(wl.B):
        k, v = res["cache"].gather(bi, 0, wl.L + wl.T + wl.S)
        ck = np.concatenate([ref["cache_k"][bi], oracle.rope_bf16(h.to64(inp["k_query"][bi]), h.to64(inp["pos_query"][bi]).astype(np.int64), wl.theta)])
        # Roped K: both sides rotate in float64 and round once to bf16, so the values
        # agree except where sin/cos differ in the last float64 bit right at a bf16
        # rounding boundary (expected count ~0); allow a handful of one-step flips.
        kg = h.to64(k[: wl.L + wl.T])
        diff = np.abs(kg - ck)
        worst = np.unravel_index(np.argmax(diff), diff.shape)
        assert np.all(diff <= np.abs(ck) * 2.0 ** -7), f"cache K off at {worst}: gpu {kg[worst]} oracle {ck[worst]}"
        assert np.count_nonzero(diff) <= 4, f"cache K differs in {np.count_nonzero(diff)} elements"
        assert np.array_equal(h.to64(v[: wl.L]), ref["cache_v"][bi]), "cache V must be a bit-exact copy"
    h.assert_out(res["o_part"], ref["o_part"], "phase2 partial O")
    h.assert_lse(res["lse_part"], ref["lse_part"], "phase2 partial LSE")
    h.assert_out(res["o_query"], ref["o_query"], "merged query O")
    h.assert_lse(res["lse_query"], ref["lse_query"], "merged query LSE")
    h.assert_out(res["o_dec"][:, :, 0], ref["o_dec"], "decode O")
    h.assert_lse(res["lse_dec"], ref["lse_dec"], "decode LSE")
    return res


@pytest.mark.parametrize("name", list(SMALL))
def test_full_path_matches_oracle(name):
    _full_compare(SMALL[name])


def test_permuted_page_table_is_bit_identical():
    """A scattered physical page assignment changes no result bit."""
    h = H()
    wl = SMALL["d128-g4-b2"]
    inp = make_inputs(wl, "cuda")
    base = h.run_gpu(wl, inp)
    max_pages = base["cache"].max_pages
    perm = torch.randperm(wl.B * max_pages + 7, generator=torch.Generator().manual_seed(3))[: wl.B * max_pages]
    pt = perm.view(wl.B, max_pages).to(torch.int32)
    other = h.run_gpu(wl, inp, page_table=pt, num_pages=wl.B * max_pages + 7)
    for key in ("o_ctx", "o_part", "lse_part", "o_query", "lse_query", "o_dec", "lse_dec"):
        assert torch.equal(base[key], other[key]), key


def test_build_positions_bit_exact():
    import block_sparse_attention_star_b200 as star
    h = H()
    for wl, offset in ((get_config("tiny"), 0), (SMALL["d128-g4-b2"], 1000)):
        shape = h.shape_of(wl)
        cache = star.PagedKVCache(shape)
        pos = (torch.arange(wl.L, dtype=torch.int32) + offset).repeat(wl.B, 1).cuda().contiguous()
        aug = torch.empty((wl.B, wl.L + (wl.n - 1) * wl.b), dtype=torch.int32, device="cuda")
        bmap = torch.empty((wl.B, wl.L, 3), dtype=torch.int32, device="cuda")
        star.star_build_positions(shape, cache, pos, aug, bmap)
        torch.cuda.synchronize()
        for bi in range(wl.B):
            blocks = oracle.augmented_context(wl.L, wl.b, pos[bi].cpu().numpy())
            want = np.concatenate([blk["pos"] for blk in blocks])
            assert np.array_equal(aug[bi].cpu().numpy(), want)
            want_map = oracle.block_map(wl.L, wl.b, wl.page_tokens, cache.page_table[bi].cpu().numpy())
            assert np.array_equal(bmap[bi].cpu().numpy(), want_map)


@pytest.mark.parametrize("n", [5, 37, 64])
def test_lse_merge_edge_cases(n):
    """n = 5: one warp per row; 37 and 64 partials: the decode-sized variant (two warps per row)."""
    import block_sparse_attention_star_b200 as star
    rng = np.random.default_rng(5 + n)
    for d in (64, 128):
        rows = 300
        O = rng.standard_normal((n, rows, d)).astype(np.float32)
        L = (rng.standard_normal((n, rows)) * 20).astype(np.float32)
        L[1, :50] = -np.inf                  # empty blocks
        L[:, 60] = -np.inf                   # a row with no usable partial
        L[0, 70:80] = 1e4                    # differences far beyond exp's range
        L[2, 80:90] = np.nan                 # filtered like an empty block, and reported
        O[1, :50] = np.nan                   # an empty partial's O (0/0) must not leak into the sum
        out = torch.empty((rows, d), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(rows, dtype=torch.float32, device="cuda")
        star.star_lse_merge(n, rows, d, torch.from_numpy(O).cuda(), torch.from_numpy(L).cuda(), out, lse)
        with pytest.raises(star.StarError) as e:
            star.star_device_status()
        assert e.value.code == star.STAR_ERR_INVALID_ARG and "NaN or +inf" in str(e.value)
        assert star.star_device_status() == 0          # read and cleared
        ref_o, ref_l = oracle.lse_merge(O.astype(np.float64), L.astype(np.float64))
        h = H()
        h.assert_out(out, ref_o, "merge O")
        g = lse.cpu().numpy()
        assert np.isneginf(g[60]) and np.all(out[60].float().cpu().numpy() == 0)
        fin = np.isfinite(ref_l)
        assert np.all(np.abs(g[fin] - ref_l[fin]) <= 1e-3 * np.maximum(1.0, np.abs(ref_l[fin]) / 1e3))
        # Without the NaN partials (-inf and huge differences only) nothing is reported.
        L2 = np.where(np.isnan(L), -np.inf, L).astype(np.float32)
        star.star_lse_merge(n, rows, d, torch.from_numpy(O).cuda(), torch.from_numpy(L2).cuda(), out, lse)
        assert star.star_device_status() == 0
        assert torch.isfinite(out.float()).all()


def test_invalid_arguments_launch_nothing():
    import block_sparse_attention_star_b200 as star
    h = H()
    wl = get_config("tiny")
    shape = h.shape_of(wl)
    cache = star.PagedKVCache(shape)
    inp = make_inputs(wl, "cuda", parts=("ctx",))
    out = torch.zeros_like(inp["q_ctx"])
    with pytest.raises(star.StarError) as e:
        star.star_phase1_encode(shape, cache, inp["q_ctx"], inp["k_ctx"], None, inp["pos_ctx"], out)
    assert e.value.code == star.STAR_ERR_INVALID_ARG
    mis = torch.empty(out.numel() + 8, dtype=torch.bfloat16, device="cuda")[1: 1 + out.numel()].view(out.shape)
    with pytest.raises(star.StarError) as e:
        star.star_phase1_encode(shape, cache, inp["q_ctx"], inp["k_ctx"], inp["v_ctx"], inp["pos_ctx"], mis)
    assert e.value.code == star.STAR_ERR_ALIGNMENT
    bad = h.shape_of(dataclasses.replace(wl, Hq=6, Hkv=2))
    with pytest.raises(star.StarError) as e:
        star.star_phase1_encode(bad, cache, inp["q_ctx"], inp["k_ctx"], inp["v_ctx"], inp["pos_ctx"], out)
    assert e.value.code == star.STAR_ERR_UNSUPPORTED_SHAPE
    small = star.StarCache(cache.c.k_pool, cache.c.v_pool, cache.c.page_table, 1, cache.num_pages)
    cache.c, saved = small, cache.c
    with pytest.raises(star.StarError) as e:
        star.star_phase1_encode(shape, cache, inp["q_ctx"], inp["k_ctx"], inp["v_ctx"], inp["pos_ctx"], out)
    assert e.value.code == star.STAR_ERR_CAPACITY
    cache.c = saved
    torch.cuda.synchronize()
    assert torch.count_nonzero(out) == 0
    assert star.star_device_status() == 0


def _decode_reference(inp, bi, ck, cv, theta):
    """Every decode step of sequence bi at once: the step-s token, roped at its position,
    attends to the cache [context, query tail, decode tokens 0..s] (oracle.global_attention
    with the rows' cache indices; the pins show the S chained decode steps equal it)."""
    h = H()
    S = inp["q_dec"].shape[0]
    dpos = inp["pos_dec"][:, bi].cpu().numpy().astype(np.int64)
    qd = oracle.rope_bf16(h.to64(inp["q_dec"][:, bi, 0]), dpos, theta)
    ck, cv = oracle.append_tail(ck, cv, h.to64(inp["k_dec"][:, bi, 0]), h.to64(inp["v_dec"][:, bi, 0]), dpos, theta)
    rows = ck.shape[0] - S + np.arange(S)
    return oracle.global_attention(qd, rows, ck, cv)


def _large_check(wl: Workload, rows_per_block: int):
    h = H()
    inp = make_inputs(wl, "cuda")
    res = h.run_gpu(wl, inp)
    assert res["status"] == 0
    rows = h.sample_rows(wl, rows_per_block)
    theta = wl.theta
    for bi in range(wl.B):
        k = h.to64(inp["k_ctx"][bi])
        v = h.to64(inp["v_ctx"][bi])
        pos = inp["pos_ctx"][bi].cpu().numpy().astype(np.int64)
        ref_rows = oracle.phase1_rows(rows, h.to64(inp["q_ctx"][bi][torch.from_numpy(rows).cuda()]), k, v, pos, wl.b, theta)
        h.assert_out(res["o_ctx"][bi][torch.from_numpy(rows).cuda()], ref_rows, f"phase1 sampled rows (seq {bi})")
        # Phase 2 and the merge: every query row, every head.
        ck = oracle.rope_bf16(k, pos, theta)
        ck, cv = oracle.append_tail(ck, v, h.to64(inp["k_query"][bi]), h.to64(inp["v_query"][bi]),
                                    inp["pos_query"][bi].cpu().numpy().astype(np.int64), theta)
        qpos = inp["pos_query"][bi].cpu().numpy().astype(np.int64)
        Op, Lp = oracle.phase2_partials(h.to64(inp["q_query"][bi]), qpos, ck, cv, wl.L, wl.b, theta)
        Oq, Lq = oracle.lse_merge(Op, Lp)
        h.assert_out(res["o_part"][:, bi], Op, "phase2 partial O")
        h.assert_lse(res["lse_part"][:, bi], Lp, "phase2 partial LSE")
        h.assert_out(res["o_query"][bi], Oq, "merged O")
        h.assert_lse(res["lse_query"][bi], Lq, "merged LSE")
        # Every decode step.
        Od, Ld = _decode_reference(inp, bi, ck, cv, theta)
        h.assert_out(res["o_dec"][:, bi, 0], Od, "decode O (every step)")
        h.assert_lse(res["lse_dec"][:, bi], Ld, "decode LSE (every step)")


def test_llama8b_32k_sampled_rows_and_full_merge():
    wl = get_config("llama8b-32k")
    _large_check(wl, 60)


def test_llama8b_128k_b32768_sampled_rows_and_full_merge():
    wl = get_config("llama8b-128k-b32768")
    _large_check(wl, 28)


@pytest.mark.parametrize("b", [4096, 8192, 16384])
def test_llama8b_128k_block_sweep_sampled(b):
    wl = get_config(f"llama8b-128k-b{b}")
    _large_check(wl, 6)


def test_llama70b_128k_sampled():
    """B = 2 sequences, GQA group 8, 128 query tokens (one full query tile per head)."""
    wl = get_config("llama70b-128k")
    _large_check(wl, 6)


def test_million_token_context_sampled_streaming_oracle():
    """1M context (8 blocks of 131072): sampled Phase-1 rows, every Phase-2 partial,
    the merged query output and every decode step, with the oracle run block by block
    (its per-block partials merged by oracle.lse_merge, exact by the merge pins) so
    host memory stays small."""
    h = H()
    wl = get_config("ctx-1m")
    inp = make_inputs(wl, "cuda")
    res = h.run_gpu(wl, inp)
    assert res["status"] == 0
    theta, b, L, T, S = wl.theta, wl.b, wl.L, wl.T, wl.S
    k = h.to64(inp["k_ctx"][0])
    v = h.to64(inp["v_ctx"][0])
    pos = inp["pos_ctx"][0].cpu().numpy().astype(np.int64)
    rows = h.sample_rows(wl, 3)
    q_rows = h.to64(inp["q_ctx"][0][torch.from_numpy(rows).cuda()])
    ref_rows = oracle.phase1_rows(rows, q_rows, k, v, pos, b, theta)
    h.assert_out(res["o_ctx"][0][torch.from_numpy(rows).cuda()], ref_rows, "1M phase1 sampled rows")
    qpos = inp["pos_query"][0].cpu().numpy().astype(np.int64)
    qr = oracle.rope_bf16(h.to64(inp["q_query"][0]), qpos, theta)
    kq = oracle.rope_bf16(h.to64(inp["k_query"][0]), qpos, theta)
    vq = h.to64(inp["v_query"][0])
    dpos = inp["pos_dec"][:, 0].cpu().numpy().astype(np.int64)
    qd = oracle.rope_bf16(h.to64(inp["q_dec"][:, 0, 0]), dpos, theta)
    kd = oracle.rope_bf16(h.to64(inp["k_dec"][:, 0, 0]), dpos, theta)
    vd = h.to64(inp["v_dec"][:, 0, 0])
    q_idx = L + np.arange(T)
    d_idx = L + T + np.arange(S)
    Op, Lp, Od, Ld = [], [], [], []
    for i in range(wl.n):
        ck = oracle.rope_bf16(k[i * b:(i + 1) * b], pos[i * b:(i + 1) * b], theta)
        cv = v[i * b:(i + 1) * b]
        key_idx = np.arange(i * b, (i + 1) * b)
        if i == wl.n - 1:                      # the tail: query tokens, then the decode tokens
            ck, cv = np.concatenate([ck, kq, kd]), np.concatenate([cv, vq, vd])
            key_idx = np.concatenate([key_idx, q_idx, d_idx])
        O, LS = oracle.attend(qr, ck, cv, key_idx[None, :] <= q_idx[:, None])
        Op.append(O)
        Lp.append(LS)
        O, LS = oracle.attend(qd, ck, cv, key_idx[None, :] <= d_idx[:, None])
        Od.append(O)
        Ld.append(LS)
    Op, Lp = np.stack(Op), np.stack(Lp)
    h.assert_out(res["o_part"][:, 0], Op, "1M phase2 partial O")
    h.assert_lse(res["lse_part"][:, 0], Lp, "1M phase2 partial LSE")
    Oq, Lq = oracle.lse_merge(Op, Lp)
    h.assert_out(res["o_query"][0], Oq, "1M merged O")
    h.assert_lse(res["lse_query"][0], Lq, "1M merged LSE")
    Odm, Ldm = oracle.lse_merge(np.stack(Od), np.stack(Ld))
    h.assert_out(res["o_dec"][:, 0, 0], Odm, "1M decode O (every step)")
    h.assert_lse(res["lse_dec"][:, 0], Ldm, "1M decode LSE (every step)")
