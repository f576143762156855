"""Pins of the oracle's whole path (``oracle.run_star``) against independent brute force.

``run_star`` chains Phase 1, the query tail append, the per-block partials, the
log-sum-exp merge, and S decode steps that each append their token's K/V and
carry the cache forward ("Star Attention 完全拆解(一)", "Phase 2: 局部注意力与本地统计
量" and "组装全局结果"; generated tokens attend to every prior cached token, per the
abstract of "Star Attention: Efficient LLM Inference over Long Sequences").  The
pins below rebuild what each output must equal without calling any of those
oracle steps:

* n = 1: Star Attention has no anchor and no split, so the whole path is one
  index-causal attention over the concatenated sequence [c, q, gen], computed
  here by one library SDPA call (the path-level form of "n = 1 equals full causal
  attention").
* n > 1: the query and decode rows attend to the cache exactly ("组装全局结果"
  proves the merge exact), so they equal one library SDPA over the explicitly
  concatenated, independently roped cache; the Phase-1 rows equal one full-length
  attention under the Star mask; each per-block partial equals SDPA over that
  block's keys.
* Two planted mistakes (decode steps that forget the tokens appended before them;
  a query tail placed before the context) are each shown to fail these pins.

RoPE here is the complex-multiplication form, and the library calls are torch
``scaled_dot_product_attention`` and ``scipy.special.logsumexp`` in float64.
"""

import numpy as np
import pytest

import oracle
from tests.test_oracle_pins import _bf16_values, lse_lib, rope_complex, sdpa, star_mask

THETA = 500000.0


def _inputs(seed, B, L, T, S, Hq, Hkv, d, k_scale=1.0):
    rng = np.random.default_rng(seed)
    f = lambda *sh, s=1.0: _bf16_values(rng, sh, s)
    return {
        "q_ctx": f(B, L, Hq, d), "k_ctx": f(B, L, Hkv, d, s=k_scale), "v_ctx": f(B, L, Hkv, d),
        "pos_ctx": np.tile(np.arange(L), (B, 1)),
        "q_query": f(B, T, Hq, d), "k_query": f(B, T, Hkv, d, s=k_scale), "v_query": f(B, T, Hkv, d),
        "pos_query": np.tile(L + np.arange(T), (B, 1)),
        "q_dec": f(S, B, 1, Hq, d), "k_dec": f(S, B, 1, Hkv, d, s=k_scale), "v_dec": f(S, B, 1, Hkv, d),
        "pos_dec": np.tile((L + T + np.arange(S))[:, None], (1, B)),
    }


def _sequence(inp, bi):
    """Sequence bi as one token stream [c, q, gen]: pre-RoPE q, k, v and position ids."""
    q = np.concatenate([inp["q_ctx"][bi], inp["q_query"][bi], inp["q_dec"][:, bi, 0]])
    k = np.concatenate([inp["k_ctx"][bi], inp["k_query"][bi], inp["k_dec"][:, bi, 0]])
    v = np.concatenate([inp["v_ctx"][bi], inp["v_query"][bi], inp["v_dec"][:, bi, 0]])
    pos = np.concatenate([inp["pos_ctx"][bi], inp["pos_query"][bi], inp["pos_dec"][:, bi]])
    return q, k, v, pos


def _roped(x, pos):
    return oracle.round_to_bf16(rope_complex(x, pos, THETA))


@pytest.mark.parametrize("B,L,T,S,Hq,Hkv,d", [(2, 48, 5, 4, 4, 2, 16), (1, 32, 1, 3, 8, 1, 8)])
def test_single_block_path_is_one_causal_attention_over_context_query_and_generation(B, L, T, S, Hq, Hkv, d):
    inp = _inputs(40 + L, B, L, T, S, Hq, Hkv, d, k_scale=2.0)
    r = oracle.run_star(inp, L, L, THETA)          # b = L: one block
    N = L + T + S
    causal = np.tril(np.ones((N, N), dtype=bool))
    for bi in range(B):
        q, k, v, pos = _sequence(inp, bi)
        qr, kr = _roped(q, pos), _roped(k, pos)
        O = sdpa(qr, kr, v, causal)
        LSE = lse_lib(qr, kr, causal)
        np.testing.assert_allclose(r["o_ctx"][bi], O[:L], rtol=0, atol=1e-12)
        np.testing.assert_allclose(r["o_query"][bi], O[L:L + T], rtol=0, atol=1e-12)
        np.testing.assert_allclose(r["lse_query"][bi], LSE[L:L + T], rtol=0, atol=1e-12)
        np.testing.assert_allclose(r["o_dec"][:, bi], O[L + T:], rtol=0, atol=1e-12)
        np.testing.assert_allclose(r["lse_dec"][:, bi], LSE[L + T:], rtol=0, atol=1e-12)
        # One block: its partial is the whole answer.
        np.testing.assert_allclose(r["o_part"][0, bi], O[L:L + T], rtol=0, atol=1e-12)
        np.testing.assert_allclose(r["lse_part"][0, bi], LSE[L:L + T], rtol=0, atol=1e-12)
        np.testing.assert_array_equal(r["cache_k"][bi], kr[:L])
        np.testing.assert_array_equal(r["cache_v"][bi], v[:L])


def _check_multi_block(r, inp, L, b, T, S):
    """run_star's outputs against brute force over the explicit cache, per sequence."""
    for bi in range(inp["q_ctx"].shape[0]):
        q, k, v, pos = _sequence(inp, bi)
        qr, kr = _roped(q, pos), _roped(k, pos)
        # Phase 1: one full-length attention under the Star mask; the cache holds every
        # context token once, roped at its own position.
        O1 = sdpa(qr[:L], kr[:L], v[:L], star_mask(L, b))
        np.testing.assert_allclose(r["o_ctx"][bi], O1, rtol=0, atol=1e-12)
        np.testing.assert_array_equal(r["cache_k"][bi], kr[:L])
        np.testing.assert_array_equal(r["cache_v"][bi], v[:L])
        # Query and decode rows: exact attention over the cache [c, q, gen] up to themselves.
        N = L + T + S
        rows = np.arange(L, N)
        mask = np.arange(N)[None, :] <= rows[:, None]
        O = sdpa(qr[L:], kr, v, mask)
        LSE = lse_lib(qr[L:], kr, mask)
        np.testing.assert_allclose(r["o_query"][bi], O[:T], rtol=0, atol=1e-12)
        np.testing.assert_allclose(r["lse_query"][bi], LSE[:T], rtol=0, atol=1e-12)
        np.testing.assert_allclose(r["o_dec"][:, bi], O[T:], rtol=0, atol=1e-12)
        np.testing.assert_allclose(r["lse_dec"][:, bi], LSE[T:], rtol=0, atol=1e-12)
        # Per-block partials of the query rows: block i's keys, the last block with the tail.
        n = L // b
        for i in range(n):
            lo, hi = i * b, (i + 1) * b if i < n - 1 else L + T
            m = np.zeros((T, N), dtype=bool)
            m[:, lo:hi] = mask[:T, lo:hi]
            np.testing.assert_allclose(r["o_part"][i, bi], sdpa(qr[L:L + T], kr, v, m), rtol=0, atol=1e-12)
            np.testing.assert_allclose(r["lse_part"][i, bi], lse_lib(qr[L:L + T], kr, m), rtol=0, atol=1e-12)


@pytest.mark.parametrize("B,L,b,T,S,Hq,Hkv,d", [(2, 64, 16, 3, 4, 4, 2, 16), (1, 96, 32, 6, 3, 8, 2, 8)])
def test_multi_block_path_equals_brute_force_over_the_explicit_cache(B, L, b, T, S, Hq, Hkv, d):
    inp = _inputs(50 + L + b, B, L, T, S, Hq, Hkv, d, k_scale=2.0)
    r = oracle.run_star(inp, L, b, THETA)
    _check_multi_block(r, inp, L, b, T, S)


def _path_pins_hold(seed=60):
    B, L, b, T, S, Hq, Hkv, d = 1, 64, 16, 4, 3, 4, 2, 16
    inp = _inputs(seed, B, L, T, S, Hq, Hkv, d, k_scale=2.0)
    try:
        _check_multi_block(oracle.run_star(inp, L, b, THETA), inp, L, b, T, S)
        return True
    except AssertionError:
        return False


def test_path_pins_hold_unplanted():
    assert _path_pins_hold()


def test_planted_decode_that_does_not_carry_the_cache_is_caught(monkeypatch):
    real = oracle.star_oracle.decode_step

    def forgetful(q_tok, k_tok, v_tok, pos, ck, cv, theta):
        O, LSE, _, _ = real(q_tok, k_tok, v_tok, pos, ck, cv, theta)
        return O, LSE, ck, cv                       # the next step loses this token's K/V

    monkeypatch.setattr(oracle.star_oracle, "decode_step", forgetful)
    assert not _path_pins_hold()


def test_planted_query_tail_before_the_context_is_caught(monkeypatch):
    real = oracle.star_oracle.append_tail

    def prepend_query(ck, cv, k_new, v_new, pos_new, theta):
        if k_new.shape[0] > 1:                      # the query tail (decode appends one token)
            tk, tv = real(ck[:0], cv[:0], k_new, v_new, pos_new, theta)
            return np.concatenate([tk, ck]), np.concatenate([tv, cv])
        return real(ck, cv, k_new, v_new, pos_new, theta)

    monkeypatch.setattr(oracle.star_oracle, "append_tail", prepend_query)
    assert not _path_pins_hold()


def test_variable_length_path_equals_brute_force_per_sequence():
    """Per-sequence context lengths: each sequence's outputs equal the brute force over its
    own [c, q, gen] (its tail starting at its own length), padded rows excluded."""
    L, b, T, S, Hq, Hkv, d = 64, 16, 3, 2, 4, 2, 16
    lens = [64, 37, 16]
    inp = _inputs(70, len(lens), L, T, S, Hq, Hkv, d, k_scale=2.0)
    inp["seq_len"] = np.array(lens)
    inp["pos_query"] = np.stack([Ls + np.arange(T) for Ls in lens])
    inp["pos_dec"] = np.stack([[Ls + T + s for Ls in lens] for s in range(S)])
    r = oracle.run_star(inp, L, b, THETA)
    for bi, Ls in enumerate(lens):
        q = np.concatenate([inp["q_ctx"][bi][:Ls], inp["q_query"][bi], inp["q_dec"][:, bi, 0]])
        k = np.concatenate([inp["k_ctx"][bi][:Ls], inp["k_query"][bi], inp["k_dec"][:, bi, 0]])
        v = np.concatenate([inp["v_ctx"][bi][:Ls], inp["v_query"][bi], inp["v_dec"][:, bi, 0]])
        pos = np.concatenate([inp["pos_ctx"][bi][:Ls], inp["pos_query"][bi], inp["pos_dec"][:, bi]])
        qr, kr = _roped(q, pos), _roped(k, pos)
        N = Ls + T + S
        # Phase 1 with a ragged last block: Star mask over the sequence's own length.
        t = np.arange(Ls)
        same = (t[:, None] // b) == (t[None, :] // b)
        caus = t[None, :] <= t[:, None]
        smask = (same & caus) | ((t[None, :] < b) & (t[:, None] >= b))
        np.testing.assert_allclose(r["o_ctx"][bi][:Ls], sdpa(qr[:Ls], kr[:Ls], v[:Ls], smask), rtol=0, atol=1e-12)
        rows = np.arange(Ls, N)
        mask = np.arange(N)[None, :] <= rows[:, None]
        O, LSE = sdpa(qr[Ls:], kr, v, mask), lse_lib(qr[Ls:], kr, mask)
        np.testing.assert_allclose(r["o_query"][bi], O[:T], rtol=0, atol=1e-12)
        np.testing.assert_allclose(r["lse_query"][bi], LSE[:T], rtol=0, atol=1e-12)
        np.testing.assert_allclose(r["o_dec"][:, bi], O[T:], rtol=0, atol=1e-12)
        np.testing.assert_allclose(r["lse_dec"][:, bi], LSE[T:], rtol=0, atol=1e-12)
