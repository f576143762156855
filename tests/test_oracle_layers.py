"""Pins of the oracle's multi-layer Phase 1 (``oracle.encode_layers``).

[SA1] "仓库里的真实实现": every augmented block [anchor; c_i] runs the whole model
forward on its own and the anchor's part of every layer is dropped.  The oracle
instead makes one pass over the L real tokens per layer and takes the anchor's keys
and values of each layer from that layer's block 1.  The pins run the literal
per-block forward (written here with library SDPA for the attention) and require the
same result; with one block, that is a textbook stack of causal attention layers.
"""

import numpy as np
import pytest
import torch

import oracle

THETA = 500000.0


def _model(rng, n_layers, hidden, Hq, Hkv, d):
    """A small random model: per layer q/k/v projections and an output projection with
    a residual, every result rounded to bf16 as a bf16 model would."""
    layers = []
    for _ in range(n_layers):
        wq = oracle.round_to_bf16(rng.standard_normal((hidden, Hq * d)) / np.sqrt(hidden))
        wk = oracle.round_to_bf16(rng.standard_normal((hidden, Hkv * d)) / np.sqrt(hidden))
        wv = oracle.round_to_bf16(rng.standard_normal((hidden, Hkv * d)) / np.sqrt(hidden))
        wo = oracle.round_to_bf16(rng.standard_normal((Hq * d, hidden)) / np.sqrt(Hq * d))

        def qkv(x, wq=wq, wk=wk, wv=wv):
            n = x.shape[0]
            return (oracle.round_to_bf16(x @ wq).reshape(n, Hq, d), oracle.round_to_bf16(x @ wk).reshape(n, Hkv, d),
                    oracle.round_to_bf16(x @ wv).reshape(n, Hkv, d))

        def out(x, o, wo=wo):
            return oracle.round_to_bf16(x + o.reshape(o.shape[0], -1) @ wo)

        layers.append((qkv, out))
    return layers


def _sdpa_causal(qr, kr, v):
    """Causal softmax attention by torch (float64), GQA by repeating K/V heads."""
    G = qr.shape[1] // kr.shape[1]
    q = torch.from_numpy(qr).permute(1, 0, 2)
    k = torch.from_numpy(np.repeat(kr, G, axis=1)).permute(1, 0, 2)
    vv = torch.from_numpy(np.repeat(v, G, axis=1)).permute(1, 0, 2)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, vv, is_causal=True)
    return o.permute(1, 0, 2).numpy()


def _literal(x0, pos, b, layers, a):
    """Each augmented block through all layers on its own; the anchor rows are dropped."""
    L = x0.shape[0]
    out = np.zeros_like(x0)
    for i in range(L // b):
        own = np.arange(i * b, (i + 1) * b)
        idx = own if i == 0 else np.concatenate([np.arange(a), own])
        xa, pa = x0[idx], pos[idx]
        for qkv, proj in layers:
            q, k, v = qkv(xa)
            o = _sdpa_causal(oracle.rope_bf16(q, pa, THETA), oracle.rope_bf16(k, pa, THETA), v)
            xa = proj(xa, oracle.round_to_bf16(o))
        out[own] = xa[len(idx) - b:]
    return out


@pytest.mark.parametrize("L,b,a,n_layers", [(16, 4, None, 3), (16, 4, 2, 3), (8, 8, None, 2), (24, 8, 4, 2)])
def test_encode_layers_equals_the_literal_per_block_forward(L, b, a, n_layers):
    rng = np.random.default_rng(7 + L + b + (a or 0))
    Hq, Hkv, d = 4, 2, 8
    hidden = 24
    x0 = oracle.round_to_bf16(rng.standard_normal((L, hidden)))
    pos = np.arange(L)
    layers = _model(rng, n_layers, hidden, Hq, Hkv, d)
    x, per_layer = oracle.encode_layers(x0, pos, b, THETA, layers, a)
    np.testing.assert_allclose(x, _literal(x0, pos, b, layers, a if a else b), rtol=0, atol=1e-9)
    assert len(per_layer) == n_layers


def test_encode_layers_catches_planted_mistakes(monkeypatch):
    """Plausible mistakes must fail the literal comparison: the attention output not
    rounded to bf16 before the next layer, and an anchor of the wrong size."""
    import sys

    L, b, Hq, Hkv, d, hidden = 16, 4, 4, 2, 8, 24
    rng = np.random.default_rng(3)
    x0 = oracle.round_to_bf16(rng.standard_normal((L, hidden)))
    pos = np.arange(L)
    layers = _model(rng, 2, hidden, Hq, Hkv, d)
    ref = _literal(x0, pos, b, layers, b)

    x, _ = oracle.encode_layers(x0, pos, b, THETA, layers, 2)  # anchor of 2 tokens instead of b
    assert np.max(np.abs(x - ref)) > 1e-3

    real_round = oracle.star_oracle.round_to_bf16

    def round_except_in_encode_layers(v):
        return v if sys._getframe(1).f_code.co_name == "encode_layers" else real_round(v)

    monkeypatch.setattr(oracle.star_oracle, "round_to_bf16", round_except_in_encode_layers)
    x, _ = oracle.star_oracle.encode_layers(x0, pos, b, THETA, layers)
    assert np.max(np.abs(x - ref)) > 1e-6
