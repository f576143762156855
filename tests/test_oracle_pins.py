"""Pins of the CPU oracle to things other than itself.

Each test checks an oracle function against a closed form, a library routine
(torch scaled_dot_product_attention, scipy logsumexp, torch's bf16 cast), an
independent reformulation, or a fixture enumerated by hand from the pages.
The mutation tests at the end plant a plausible mistake in the oracle (on the
CPU, through monkeypatch) and show that a pin catches it.
"""

import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _bf16_values(rng, shape, scale=1.0):
    return oracle.round_to_bf16(rng.standard_normal(shape) * scale)


# ---------------------------------------------------------------------------
# Independent routes used by several pins
# ---------------------------------------------------------------------------

def rope_complex(x, pos, theta):
    """RoPE as complex multiplication: (x_j + i x_{j+d/2}) * exp(i pos theta^(-2j/d))."""
    d = x.shape[-1]
    freq = 1.0 / (theta ** (np.arange(0, d, 2, dtype=np.float64) / d))
    z = x[..., : d // 2] + 1j * x[..., d // 2:]
    rot = np.exp(1j * np.asarray(pos, dtype=np.float64)[:, None, None] * freq[None, None, :])
    w = z * rot
    return np.concatenate([w.real, w.imag], axis=-1)


def sdpa(q, k, v, mask):
    """Library attention in fp64: q [M, Hq, d], k/v [N, Hkv, d], mask bool [M, N]."""
    G = q.shape[1] // k.shape[1]
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    kt = torch.from_numpy(np.repeat(k, G, axis=1)).permute(1, 0, 2)[None]
    vt = torch.from_numpy(np.repeat(v, G, axis=1)).permute(1, 0, 2)[None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.from_numpy(mask))
    return o[0].permute(1, 0, 2).numpy()


def lse_lib(q, k, mask):
    """log sum exp(q.k/sqrt(d)) over visible keys via scipy.special.logsumexp."""
    G = q.shape[1] // k.shape[1]
    d = q.shape[-1]
    out = np.zeros(q.shape[:2])
    for h in range(q.shape[1]):
        s = np.einsum("md,nd->mn", q[:, h], k[:, h // G]) / math.sqrt(d)
        out[:, h] = scipy.special.logsumexp(np.where(mask, s, -np.inf), axis=1)
    return out


def star_mask(L, b):
    """Full-length visibility of Phase 1: anchor keys plus own block up to the row."""
    t = np.arange(L)
    same_block = (t[:, None] // b) == (t[None, :] // b)
    causal = t[None, :] <= t[:, None]
    anchor = t[None, :] < b
    return (anchor & causal) | (same_block & causal) | (anchor & (t[:, None] >= b))


def full_star_phase1(q, k, v, pos, b, theta):
    """Phase 1 as ONE full-length attention with the Star mask (no c' built)."""
    qr = oracle.round_to_bf16(rope_complex(q, pos, theta))
    kr = oracle.round_to_bf16(rope_complex(k, pos, theta))
    return sdpa(qr, kr, v, star_mask(q.shape[0], b)), kr


# ---------------------------------------------------------------------------
# bf16 rounding
# ---------------------------------------------------------------------------

def test_bf16_round_hand_ties():
    u = 2.0 ** -7                       # bf16 ulp at 1.0
    cases = {
        1.0 + u / 2: 1.0,               # tie -> even (1.0)
        1.0 + 3 * u / 2: 1.0 + 2 * u,   # tie -> even (mantissa ...10)
        -(1.0 + u / 2): -1.0,
        1.0 + u / 2 + 2.0 ** -30: 1.0 + u,   # just above the tie
        1.0 + u / 2 - 2.0 ** -30: 1.0,       # just below
        3.0: 3.0,
        255.5: 256.0,                   # 8 significant bits: 255.5 is a tie between 255 and 256 -> 256 (even)
        0.1: 0.10009765625,
    }
    for x, want in cases.items():
        assert oracle.round_to_bf16(x) == want, (x, oracle.round_to_bf16(x), want)


def test_bf16_round_matches_torch_cast_on_fp32_inputs():
    rng = np.random.default_rng(1)
    x32 = (rng.standard_normal(200000) * np.exp(rng.uniform(-8, 8, 200000))).astype(np.float32)
    want = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.round_to_bf16(x32.astype(np.float64))
    assert np.array_equal(got, want)


# ---------------------------------------------------------------------------
# RoPE
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("d", [8, 64, 128])
def test_rope_matches_complex_form(d):
    rng = np.random.default_rng(2)
    x = rng.standard_normal((50, 3, d))
    pos = np.concatenate([np.arange(25), rng.integers(0, 1 << 20, 25)])
    got = oracle.apply_rope(x, pos, 500000.0)
    want = rope_complex(x, pos, 500000.0)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-9)


def test_rope_closed_form_angles_and_identity():
    inv = oracle.rope_inv_freq(4, 10000.0)
    np.testing.assert_allclose(inv, [1.0, 0.01], rtol=1e-15)
    np.testing.assert_allclose(oracle.rope_angles([3], 4, 10000.0), [[3.0, 0.03]], rtol=1e-15)
    # e_0 at position p turns into (cos p, ..., sin p, ...) for the j=0 pair.
    e0 = np.zeros((1, 1, 4)); e0[0, 0, 0] = 1.0
    y = oracle.apply_rope(e0, [3], 10000.0)
    np.testing.assert_allclose(y[0, 0], [math.cos(3.0), 0.0, math.sin(3.0), 0.0], atol=1e-15)
    x = np.random.default_rng(3).standard_normal((4, 2, 16))
    assert np.array_equal(oracle.apply_rope(x, np.zeros(4), 500000.0), x)


def test_rope_norm_and_relative_shift():
    rng = np.random.default_rng(4)
    d = 64
    q = rng.standard_normal((20, 1, d))
    k = rng.standard_normal((20, 1, d))
    pq = rng.integers(0, 100000, 20)
    pk = rng.integers(0, 100000, 20)
    rq = oracle.apply_rope(q, pq, 500000.0)
    pairs_in = q[..., : d // 2] ** 2 + q[..., d // 2:] ** 2
    pairs_out = rq[..., : d // 2] ** 2 + rq[..., d // 2:] ** 2
    np.testing.assert_allclose(pairs_out, pairs_in, rtol=1e-12)
    s0 = np.einsum("nd,nd->n", rq[:, 0], oracle.apply_rope(k, pk, 500000.0)[:, 0])
    for shift in (1, 4096, 700000):
        s1 = np.einsum("nd,nd->n", oracle.apply_rope(q, pq + shift, 500000.0)[:, 0],
                       oracle.apply_rope(k, pk + shift, 500000.0)[:, 0])
        np.testing.assert_allclose(s1, s0, rtol=0, atol=1e-9)


# ---------------------------------------------------------------------------
# c' construction, position ids, KV drop, block map (hand fixture)
# ---------------------------------------------------------------------------

def test_augmented_context_matches_hand_fixture():
    g = _golden("positions_L8_b2.json")
    blocks = oracle.augmented_context(g["L"], g["b"], g["pos_ctx"])
    assert [blk["tokens"].tolist() for blk in blocks] == g["augmented_tokens"]
    assert [blk["pos"].tolist() for blk in blocks] == g["augmented_pos"]
    assert sum(len(blk["tokens"]) for blk in blocks) == g["augmented_total"]
    dropped = sum(len(blk["tokens"]) - len(blk["kept"]) for blk in blocks)
    assert dropped == g["anchor_rows_dropped"]
    kept = np.concatenate([blk["tokens"][blk["kept"]] for blk in blocks])
    assert kept.tolist() == g["cached_tokens"]
    off = oracle.augmented_context(g["L"], g["b"], g["offset_pos_ctx"])
    assert [blk["pos"].tolist() for blk in off] == g["offset_augmented_pos"]


def test_block_map_matches_hand_fixture():
    g = _golden("positions_L8_b2.json")
    bm = oracle.block_map(g["L"], g["b"], g["page_tokens"], g["page_table"])
    assert bm.tolist() == g["block_map"]


def test_star_mask_rule_matches_hand_fixture():
    g = _golden("positions_L8_b2.json")
    assert star_mask(g["L"], g["b"]).astype(int).tolist() == g["star_visibility"]


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------

def test_causal_attention_matches_library():
    rng = np.random.default_rng(5)
    q = _bf16_values(rng, (40, 4, 16))
    k = _bf16_values(rng, (40, 2, 16))
    v = _bf16_values(rng, (40, 2, 16))
    O, LSE = oracle.causal_attention(q, k, v)
    mask = np.tril(np.ones((40, 40), dtype=bool))
    np.testing.assert_allclose(O, sdpa(q, k, v, mask), rtol=0, atol=1e-12)
    np.testing.assert_allclose(LSE, lse_lib(q, k, mask), rtol=0, atol=1e-12)


def test_phase1_single_block_is_causal_attention():
    """n = 1: no anchor, Phase 1 is plain causal attention over the roped context."""
    rng = np.random.default_rng(6)
    L, theta = 64, 500000.0
    q, k, v = _bf16_values(rng, (L, 4, 16)), _bf16_values(rng, (L, 2, 16)), _bf16_values(rng, (L, 2, 16))
    pos = np.arange(L)
    O, ck, cv = oracle.phase1(q, k, v, pos, L, theta)
    qr = oracle.round_to_bf16(rope_complex(q, pos, theta))
    kr = oracle.round_to_bf16(rope_complex(k, pos, theta))
    np.testing.assert_allclose(O, sdpa(qr, kr, v, np.tril(np.ones((L, L), dtype=bool))), atol=1e-12)
    assert np.array_equal(ck, kr) and np.array_equal(cv, v)


@pytest.mark.parametrize("L,b", [(96, 32), (256, 64), (128, 16)])
def test_phase1_equals_full_length_star_mask(L, b):
    """Literal c' construction == one full-length attention with the Star mask."""
    rng = np.random.default_rng(7 + L + b)
    theta = 500000.0
    q, k, v = _bf16_values(rng, (L, 4, 16)), _bf16_values(rng, (L, 2, 16), 3.0), _bf16_values(rng, (L, 2, 16))
    pos = np.arange(L)
    O, ck, cv = oracle.phase1(q, k, v, pos, b, theta)
    O_ref, kr = full_star_phase1(q, k, v, pos, b, theta)
    np.testing.assert_allclose(O, O_ref, rtol=0, atol=1e-12)
    # The cache holds each token once: roped at its own position (anchor copies dropped).
    assert ck.shape == k.shape and np.array_equal(ck, kr) and np.array_equal(cv, v)


def test_phase1_rows_equal_full_length_star_mask():
    rng = np.random.default_rng(8)
    L, b, theta = 192, 64, 500000.0
    q, k, v = _bf16_values(rng, (L, 4, 16)), _bf16_values(rng, (L, 2, 16)), _bf16_values(rng, (L, 2, 16))
    rows = np.array([0, 5, 63, 64, 100, 127, 128, 191])
    got = oracle.phase1_rows(rows, q[rows], k, v, None, b, theta)
    O_ref, _ = full_star_phase1(q, k, v, np.arange(L), b, theta)
    np.testing.assert_allclose(got, O_ref[rows], rtol=0, atol=1e-12)


def _phase2_case(seed, L=96, b=32, T=5, Hq=4, Hkv=2, d=16):
    rng = np.random.default_rng(seed)
    theta = 500000.0
    k_ctx = _bf16_values(rng, (L, Hkv, d), 2.0)
    v_ctx = _bf16_values(rng, (L, Hkv, d))
    ck = oracle.round_to_bf16(rope_complex(k_ctx, np.arange(L), theta))
    cv = v_ctx
    qq, kq, vq = _bf16_values(rng, (T, Hq, d)), _bf16_values(rng, (T, Hkv, d)), _bf16_values(rng, (T, Hkv, d))
    pos_q = L + np.arange(T)
    return dict(L=L, b=b, T=T, theta=theta, ck=ck, cv=cv, qq=qq, kq=kq, vq=vq, pos_q=pos_q)


def test_lse_merge_of_partials_equals_brute_force():
    c = _phase2_case(9)
    ck, cv = oracle.append_tail(c["ck"], c["cv"], c["kq"], c["vq"], c["pos_q"], c["theta"])
    Op, Lp = oracle.phase2_partials(c["qq"], c["pos_q"], ck, cv, c["L"], c["b"], c["theta"])
    O, LSE = oracle.lse_merge(Op, Lp)
    qr = oracle.round_to_bf16(rope_complex(c["qq"], c["pos_q"], c["theta"]))
    kr_tail = oracle.round_to_bf16(rope_complex(c["kq"], c["pos_q"], c["theta"]))
    K = np.concatenate([c["ck"], kr_tail])
    V = np.concatenate([c["cv"], c["vq"]])
    mask = np.arange(K.shape[0])[None, :] <= (c["L"] + np.arange(c["T"]))[:, None]
    np.testing.assert_allclose(O, sdpa(qr, K, V, mask), rtol=0, atol=1e-12)
    np.testing.assert_allclose(LSE, lse_lib(qr, K, mask), rtol=0, atol=1e-12)
    assert Op.shape[0] == c["L"] // c["b"]


def test_lse_merge_identities_and_overflow():
    rng = np.random.default_rng(10)
    O = rng.standard_normal((4, 6, 8))
    L = rng.standard_normal((4, 6)) * 5
    one_O, one_L = oracle.lse_merge(O[:1], L[:1])
    assert np.array_equal(one_O, O[0]) and np.array_equal(one_L, L[0])
    # Order does not matter; grouping does not matter.
    a = oracle.lse_merge(O, L)
    b = oracle.lse_merge(O[::-1], L[::-1])
    np.testing.assert_allclose(a[0], b[0], atol=1e-13)
    np.testing.assert_allclose(a[1], b[1], atol=1e-13)
    left = oracle.lse_merge(O[:2], L[:2])
    right = oracle.lse_merge(O[2:], L[2:])
    c = oracle.lse_merge(np.stack([left[0], right[0]]), np.stack([left[1], right[1]]))
    np.testing.assert_allclose(c[0], a[0], atol=1e-13)
    np.testing.assert_allclose(c[1], a[1], atol=1e-13)
    # Closed form: weights are softmax(LSE) over the partials.
    w = np.exp(L - scipy.special.logsumexp(L, axis=0))
    np.testing.assert_allclose(a[0], np.einsum("pr,prd->rd", w, O), atol=1e-13)
    # A -inf partial is the identity; an all-empty row gives (0, -inf).
    Lm = L.copy(); Lm[2, :] = -np.inf
    d1 = oracle.lse_merge(O, Lm)
    d2 = oracle.lse_merge(np.delete(O, 2, 0), np.delete(L, 2, 0))
    np.testing.assert_allclose(d1[0], d2[0], atol=1e-13)
    Le = np.full_like(L, -np.inf)
    e = oracle.lse_merge(O, Le)
    assert np.all(e[0] == 0) and np.all(e[1] == -np.inf)
    # NaN partial is filtered like an empty block.
    Ln = L.copy(); Ln[1, :] = np.nan
    f = oracle.lse_merge(O, Ln)
    g = oracle.lse_merge(np.delete(O, 1, 0), np.delete(L, 1, 0))
    np.testing.assert_allclose(f[0], g[0], atol=1e-13)
    # Differences far beyond exp's range: the dominant partial wins, nothing overflows.
    Lb = np.array([[1000.0], [-1000.0], [0.0]])
    Ob = np.array([[[1.0, 2.0]], [[3.0, 4.0]], [[5.0, 6.0]]])
    h = oracle.lse_merge(Ob, Lb)
    assert np.all(np.isfinite(h[0])) and np.allclose(h[0], [[1.0, 2.0]]) and np.isclose(h[1][0], 1000.0)


def test_decode_step_attends_to_whole_cache_and_itself():
    c = _phase2_case(11, T=3)
    rng = np.random.default_rng(12)
    q1, k1, v1 = _bf16_values(rng, (1, 4, 16)), _bf16_values(rng, (1, 2, 16)), _bf16_values(rng, (1, 2, 16))
    pos = c["L"] + 7
    O, LSE, ck2, cv2 = oracle.decode_step(q1, k1, v1, pos, c["ck"], c["cv"], c["theta"])
    qr = oracle.round_to_bf16(rope_complex(q1, [pos], c["theta"]))
    kr = oracle.round_to_bf16(rope_complex(k1, [pos], c["theta"]))
    K = np.concatenate([c["ck"], kr])
    V = np.concatenate([c["cv"], v1])
    mask = np.ones((1, K.shape[0]), dtype=bool)
    np.testing.assert_allclose(O, sdpa(qr, K, V, mask), atol=1e-12)
    np.testing.assert_allclose(LSE, lse_lib(qr, K, mask), atol=1e-12)
    assert ck2.shape[0] == c["L"] + 1


def test_softmax_sanity_constant_values_and_convex_hull():
    rng = np.random.default_rng(13)
    q = _bf16_values(rng, (30, 2, 16), 4.0)
    k = _bf16_values(rng, (30, 1, 16), 4.0)
    v = np.full((30, 1, 16), 2.5)
    O, _ = oracle.causal_attention(q, k, v)
    np.testing.assert_allclose(O, 2.5, atol=1e-12)
    v = _bf16_values(rng, (30, 1, 16))
    O, _ = oracle.causal_attention(q, k, v)
    assert np.all(O <= v.max(axis=0) + 1e-12) and np.all(O >= v.min(axis=0) - 1e-12)


def test_byte_accounting_matches_printed_numbers():
    g = _golden("page_numbers.json")
    kv = g["kv_bytes_per_token"]
    per_tok = oracle.kv_bytes_per_token(kv["layers"], kv["kv_heads"], kv["head_dim"], kv["bytes"])
    assert per_tok == kv["expect"]
    assert per_tok * 131072 == g["kv_bytes_128k_gib"] * 2 ** 30
    c1 = g["comm_per_host_layer_token"]
    assert oracle.phase2_comm_bytes(1, 1, 1, c1["heads"], c1["head_dim"], c1["bytes"]) == c1["expect"]
    ct = g["comm_total"]
    tot = oracle.phase2_comm_bytes(ct["hosts"], ct["layers"], ct["tokens"], ct["heads"], ct["head_dim"], ct["bytes"])
    assert round(tot / 1e9, 2) == ct["expect_gb"]


def test_run_star_shapes_and_consistency():
    rng = np.random.default_rng(14)
    B, L, b, T, S, Hq, Hkv, d = 2, 64, 16, 3, 2, 4, 2, 8
    inp = {
        "q_ctx": _bf16_values(rng, (B, L, Hq, d)), "k_ctx": _bf16_values(rng, (B, L, Hkv, d)),
        "v_ctx": _bf16_values(rng, (B, L, Hkv, d)), "pos_ctx": np.tile(np.arange(L), (B, 1)),
        "q_query": _bf16_values(rng, (B, T, Hq, d)), "k_query": _bf16_values(rng, (B, T, Hkv, d)),
        "v_query": _bf16_values(rng, (B, T, Hkv, d)), "pos_query": np.tile(L + np.arange(T), (B, 1)),
        "q_dec": _bf16_values(rng, (S, B, 1, Hq, d)), "k_dec": _bf16_values(rng, (S, B, 1, Hkv, d)),
        "v_dec": _bf16_values(rng, (S, B, 1, Hkv, d)), "pos_dec": np.tile((L + T + np.arange(S))[:, None], (1, B)),
    }
    r = oracle.run_star(inp, L, b, 500000.0)
    assert r["o_ctx"].shape == (B, L, Hq, d)
    assert r["o_part"].shape == (L // b, B, T, Hq, d) and r["lse_part"].shape == (L // b, B, T, Hq)
    assert r["o_query"].shape == (B, T, Hq, d) and r["o_dec"].shape == (S, B, Hq, d)
    for key in r:
        assert np.all(np.isfinite(r[key]))


# ---------------------------------------------------------------------------
# Planted mistakes: each must be caught by a pin above
# ---------------------------------------------------------------------------

def _star_pin_holds():
    try:
        test_phase1_equals_full_length_star_mask(96, 32)
        return True
    except AssertionError:
        return False


def test_planted_wrong_anchor_positions_is_caught(monkeypatch):
    real = oracle.star_oracle.augmented_context

    def shifted(L, b, pos_ctx=None, anchor=None, anchor_pos=None):
        blocks = real(L, b, pos_ctx, anchor, anchor_pos)
        for blk in blocks[1:]:
            blk["pos"] = blk["pos"].copy()
            blk["pos"][:b] += blk["i"] * b - b        # anchor placed just before c_i
        return blocks

    monkeypatch.setattr(oracle.star_oracle, "augmented_context", shifted)
    assert not _star_pin_holds()


def test_planted_missing_anchor_is_caught(monkeypatch):
    real = oracle.star_oracle.augmented_context

    def no_anchor(L, b, pos_ctx=None, anchor=None, anchor_pos=None):
        blocks = real(L, b, pos_ctx, anchor, anchor_pos)
        for blk in blocks[1:]:
            blk["tokens"], blk["pos"] = blk["tokens"][b:], blk["pos"][b:]
            blk["kept"] = np.arange(b)
        return blocks

    monkeypatch.setattr(oracle.star_oracle, "augmented_context", no_anchor)
    assert not _star_pin_holds()


def test_planted_rope_sign_error_is_caught(monkeypatch):
    def wrong(x, pos, theta):
        d = x.shape[-1]
        ang = oracle.rope_angles(pos, d, theta)[:, None, :]
        c, s = np.cos(ang), np.sin(ang)
        x1, x2 = x[..., : d // 2], x[..., d // 2:]
        return np.concatenate([x1 * c + x2 * s, x2 * c - x1 * s], axis=-1)

    monkeypatch.setattr(oracle.star_oracle, "apply_rope", wrong)
    monkeypatch.setattr(oracle, "apply_rope", wrong)
    with pytest.raises(AssertionError):
        test_rope_matches_complex_form(64)


def test_planted_merge_without_rescale_is_caught(monkeypatch):
    def naive(O_parts, LSE_parts):
        lse = scipy.special.logsumexp(LSE_parts, axis=0)
        return O_parts.sum(axis=0), lse           # forgets the e^{lse_i - lse} weights

    monkeypatch.setattr(oracle, "lse_merge", naive)
    with pytest.raises(AssertionError):
        test_lse_merge_of_partials_equals_brute_force()


# ---------------------------------------------------------------------------
# Anchor variants: anchor size a < b and the anchor's position ids
# ---------------------------------------------------------------------------

def star_mask_anchor(L, b, a):
    """Full-length visibility with an anchor of the first a tokens."""
    t = np.arange(L)
    same_block = (t[:, None] // b) == (t[None, :] // b)
    causal = t[None, :] <= t[:, None]
    return (same_block & causal) | ((t[None, :] < a) & (t[:, None] >= b))


def test_anchor_variants_match_hand_fixture():
    g = _golden("anchor_L12_b4_a2.json")
    for name, var in g["variants"].items():
        blocks = oracle.augmented_context(g["L"], g["b"], None, g["a"], var["anchor_pos"])
        assert [blk["tokens"].tolist() for blk in blocks] == g["augmented_tokens"], name
        assert [blk["pos"].tolist() for blk in blocks] == var["augmented_pos"], name
        assert [blk["kept"].tolist() for blk in blocks] == g["kept"], name
        kept = np.concatenate([blk["tokens"][blk["kept"]] for blk in blocks])
        assert kept.tolist() == g["cached_tokens"]
        assert sum(len(blk["tokens"]) - len(blk["kept"]) for blk in blocks) == g["anchor_rows_dropped"]
    assert star_mask_anchor(g["L"], g["b"], g["a"]).astype(int).tolist() == g["star_visibility"]


def _anchor_case(seed, L=48, b=16, a=8, Hq=4, Hkv=2, d=16):
    rng = np.random.default_rng(seed)
    q, k, v = _bf16_values(rng, (L, Hq, d)), _bf16_values(rng, (L, Hkv, d)), _bf16_values(rng, (L, Hkv, d))
    n = L // b
    offs = np.array([rng.integers(0, i * b - a + 1) for i in range(1, n)])
    variants = {
        "context": np.tile(np.arange(a), (n - 1, 1)),
        "offset": offs[:, None] + np.arange(a)[None, :],
        "zero": np.zeros((n - 1, a), dtype=np.int64),
    }
    return q, k, v, variants


def explicit_anchor_phase1(q, k, v, pos, b, a, anchor_pos, theta):
    """Phase 1 built per block from each row's key set: the anchor's first a keys roped at the
    anchor ids (complex-multiplication RoPE, rounded), then the block's own keys up to the row."""
    L = q.shape[0]
    out = np.zeros_like(q)
    qr = oracle.round_to_bf16(rope_complex(q, pos, theta))
    kr = oracle.round_to_bf16(rope_complex(k, pos, theta))
    for i in range(L // b):
        own = np.arange(i * b, (i + 1) * b)
        causal = np.tril(np.ones((b, b), dtype=bool))
        if i == 0:
            out[own] = sdpa(qr[own], kr[own], v[own], causal)
            continue
        ka = oracle.round_to_bf16(rope_complex(k[:a], anchor_pos[i - 1], theta))
        keys = np.concatenate([ka, kr[own]])
        vals = np.concatenate([v[:a], v[own]])
        mask = np.concatenate([np.ones((b, a), dtype=bool), causal], axis=1)
        out[own] = sdpa(qr[own], keys, vals, mask)
    return out


def test_phase1_anchor_variants_equal_explicit_key_sets():
    theta = 500000.0
    q, k, v, variants = _anchor_case(21)
    L, b, a = q.shape[0], 16, 8
    pos = np.arange(L)
    for name, apos in variants.items():
        O, ck, cv = oracle.phase1(q, k, v, pos, b, theta, a, apos)
        np.testing.assert_allclose(O, explicit_anchor_phase1(q, k, v, pos, b, a, apos, theta), rtol=0, atol=1e-12,
                                   err_msg=name)
        # the cache holds every token's own K/V, whatever the anchor
        assert np.array_equal(ck, oracle.round_to_bf16(rope_complex(k, pos, theta))) and np.array_equal(cv, v)
        rows = np.array([0, 5, 16, 17, 31, 32, 40, 47])
        Or = oracle.phase1_rows(rows, q[rows], k, v, pos, b, theta, a, apos)
        np.testing.assert_allclose(Or, O[rows], rtol=0, atol=1e-12, err_msg=name)


def test_phase1_context_anchor_of_full_size_is_the_default():
    """a = b with the anchor's own ids is the pages' default construction."""
    theta = 500000.0
    rng = np.random.default_rng(22)
    L, b = 48, 16
    q, k, v = _bf16_values(rng, (L, 4, 16)), _bf16_values(rng, (L, 2, 16)), _bf16_values(rng, (L, 2, 16))
    pos = np.arange(L)
    O0, _, _ = oracle.phase1(q, k, v, pos, b, theta)
    O1, _, _ = oracle.phase1(q, k, v, pos, b, theta, b, np.tile(np.arange(b), (L // b - 1, 1)))
    assert np.array_equal(O0, O1)
    ref, _ = full_star_phase1(q, k, v, pos, b, theta)
    np.testing.assert_allclose(O0, ref, rtol=0, atol=1e-12)


def test_phase1_anchor_positions_are_relative():
    """RoPE depends on position differences: shifting every position id (context and anchor) by
    the same amount changes the outputs only through the bf16 rounding of the rotated values."""
    theta = 500000.0
    q, k, v, variants = _anchor_case(23)
    L, b, a = q.shape[0], 16, 8
    pos = np.arange(L)
    for name, apos in variants.items():
        O, _, _ = oracle.phase1(q, k, v, pos, b, theta, a, apos)
        Os, _, _ = oracle.phase1(q, k, v, pos + 1000, b, theta, a, apos + 1000)
        err = np.abs(O - Os)
        assert err.max() < 2e-2 and err.mean() < 2e-3, (name, err.max(), err.mean())


def test_planted_anchor_mistake_is_caught(monkeypatch):
    """An oracle that ignores the anchor ids fails the explicit key-set pin for the offset and
    zero-reset variants (and only for those)."""
    theta = 500000.0
    q, k, v, variants = _anchor_case(24)
    L, b, a = q.shape[0], 16, 8
    pos = np.arange(L)
    real = oracle.augmented_context

    def ignores_anchor_pos(L_, b_, pos_ctx=None, anchor=None, anchor_pos=None):
        return real(L_, b_, pos_ctx, anchor, None)

    monkeypatch.setattr(oracle.star_oracle, "augmented_context", ignores_anchor_pos)
    for name, apos in variants.items():
        O, _, _ = oracle.star_oracle.phase1(q, k, v, pos, b, theta, a, apos)
        diff = np.abs(O - explicit_anchor_phase1(q, k, v, pos, b, a, apos, theta)).max()
        if name == "context":
            assert diff < 1e-12
        else:
            assert diff > 1e-2, (name, diff)


# ---------------------------------------------------------------------------
# Ragged last block, variable-length batches
# ---------------------------------------------------------------------------

def test_ragged_block_matches_hand_fixture():
    g = _golden("ragged_L10_b4.json")
    blocks = oracle.augmented_context(g["L"], g["b"])
    assert len(blocks) == g["n"]
    assert [blk["tokens"].tolist() for blk in blocks] == g["augmented_tokens"]
    assert [blk["pos"].tolist() for blk in blocks] == g["augmented_pos"]
    assert [blk["kept"].tolist() for blk in blocks] == g["kept"]
    kept = np.concatenate([blk["tokens"][blk["kept"]] for blk in blocks])
    assert kept.tolist() == g["cached_tokens"]


def _seq(seed, L, Hq=4, Hkv=2, d=16):
    rng = np.random.default_rng(seed)
    return _bf16_values(rng, (L, Hq, d)), _bf16_values(rng, (L, Hkv, d)), _bf16_values(rng, (L, Hkv, d))


def test_phase1_of_a_shorter_context_is_the_prefix_of_a_longer_one():
    """Row t's output depends only on the anchor and its own block up to t, so cutting
    the context at any length (a ragged last block) keeps the kept rows' outputs."""
    theta, b = 500000.0, 16
    q, k, v = _seq(31, 64)
    pos = np.arange(64)
    O_full, ck_full, _ = oracle.phase1(q, k, v, pos, b, theta)
    for Ls in (17, 40, 47, 63):
        O, ck, cv = oracle.phase1(q[:Ls], k[:Ls], v[:Ls], pos[:Ls], b, theta)
        np.testing.assert_allclose(O, O_full[:Ls], rtol=0, atol=1e-12, err_msg=str(Ls))
        assert np.array_equal(ck, ck_full[:Ls])
        rows = np.array([0, Ls // 2, Ls - 1])
        np.testing.assert_allclose(oracle.phase1_rows(rows, q[rows], k[:Ls], v[:Ls], pos[:Ls], b, theta), O[rows],
                                   rtol=0, atol=1e-12)


def test_ragged_phase2_merge_equals_brute_force_with_empty_partials():
    theta, b, T = 500000.0, 16, 5
    q, k, v = _seq(32, 40)
    qq, kq, vq = _seq(33, T)
    pos, qpos = np.arange(40), 40 + np.arange(T)
    _, ck, cv = oracle.phase1(q, k, v, pos, b, theta)
    ck, cv = oracle.append_tail(ck, cv, kq, vq, qpos, theta)
    Op, Lp = oracle.phase2_partials(qq, qpos, ck, cv, 40, b, theta, n_parts=5)
    assert Op.shape[0] == 5 and np.all(Lp[3:] == -np.inf) and np.all(Op[3:] == 0)
    O, LSE = oracle.lse_merge(Op, Lp)
    qr = oracle.round_to_bf16(rope_complex(qq, qpos, theta))
    mask = np.arange(ck.shape[0])[None, :] <= (40 + np.arange(T))[:, None]
    np.testing.assert_allclose(O, sdpa(qr, ck, cv, mask), rtol=0, atol=1e-12)
    np.testing.assert_allclose(LSE, lse_lib(qr, ck, mask), rtol=0, atol=1e-12)


def _varlen_batch(lens, L, b, T, S, seed=34):
    rng = np.random.default_rng(seed)
    B = len(lens)
    f = lambda *sh: _bf16_values(rng, sh)
    inp = {"q_ctx": f(B, L, 4, 16), "k_ctx": f(B, L, 2, 16), "v_ctx": f(B, L, 2, 16),
           "pos_ctx": np.tile(np.arange(L), (B, 1)), "seq_len": np.array(lens),
           "q_query": f(B, T, 4, 16), "k_query": f(B, T, 2, 16), "v_query": f(B, T, 2, 16),
           "pos_query": np.stack([Ls + np.arange(T) for Ls in lens]),
           "q_dec": f(S, B, 1, 4, 16), "k_dec": f(S, B, 1, 2, 16), "v_dec": f(S, B, 1, 2, 16),
           "pos_dec": np.stack([[Ls + T + s for Ls in lens] for s in range(S)])}
    return inp


def test_varlen_batch_equals_each_sequence_alone():
    theta, L, b, T, S = 500000.0, 64, 16, 3, 2
    lens = [64, 33, 16, 50]
    inp = _varlen_batch(lens, L, b, T, S)
    ref = oracle.run_star(inp, L, b, theta)
    for bi, Ls in enumerate(lens):
        one = {k: (v[bi:bi + 1] if k not in ("q_dec", "k_dec", "v_dec", "pos_dec") else v[:, bi:bi + 1])
               for k, v in inp.items() if k != "seq_len"}
        one = {k: (v[:, :Ls] if k in ("q_ctx", "k_ctx", "v_ctx", "pos_ctx") else v) for k, v in one.items()}
        alone = oracle.run_star(one, Ls, b, theta)
        np.testing.assert_array_equal(ref["o_ctx"][bi][:Ls], alone["o_ctx"][0])
        assert np.all(ref["o_ctx"][bi][Ls:] == 0)
        n = -(-Ls // b)
        np.testing.assert_array_equal(ref["o_part"][:n, bi], alone["o_part"][:, 0])
        assert np.all(ref["lse_part"][n:, bi] == -np.inf)
        for key in ("o_query", "lse_query"):
            np.testing.assert_allclose(ref[key][bi], alone[key][0], rtol=0, atol=1e-12)
        for key in ("o_dec", "lse_dec"):
            np.testing.assert_allclose(ref[key][:, bi], alone[key][:, 0], rtol=0, atol=1e-12)


def test_planted_tail_at_the_padded_end_is_caught(monkeypatch):
    """Placing a short sequence's query tail after the padded capacity instead of its own
    context end leaves a gap of keys it may not see; the brute-force pin catches it."""
    theta, b, T = 500000.0, 16, 4
    q, k, v = _seq(35, 40)
    qq, kq, vq = _seq(36, T)
    pos, qpos = np.arange(40), 40 + np.arange(T)
    _, ck, cv = oracle.phase1(q, k, v, pos, b, theta)
    ck, cv = oracle.append_tail(ck, cv, kq, vq, qpos, theta)
    qr = oracle.round_to_bf16(rope_complex(qq, qpos, theta))
    mask = np.arange(ck.shape[0])[None, :] <= (40 + np.arange(T))[:, None]
    want = sdpa(qr, ck, cv, mask)
    # wrong: the tail believed to start at 48 (the capacity 3 * b) -> rows see 8 extra keys
    Op, Lp = oracle.phase2_partials(qq, qpos, ck, cv, 48, b, theta)
    O, _ = oracle.lse_merge(Op, Lp)
    assert np.abs(O - want).max() > 1e-2

