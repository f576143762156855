"""GPU parity of star_encode_layers (several layers of Phase 1).

The caller's model is a small random bf16 one (synth.layer_inputs: per layer q, k, v
= x W and x <- x + o Wo), run by a torch callback on the library's stream between the
layers' Phase-1 launches.  Each layer is checked on its own inputs: the q, k, v the
callback produced for layer l (captured on the stream) go through the oracle's Phase 1,
and layer l's attention output and cache must match it as in the single-layer tests.
The structure across layers (one pass over the real tokens per layer, the anchor
taken from that layer's block 1) is pinned against the literal per-block forward in
tests/test_oracle_layers.py; an end-to-end float64 comparison of the final hidden
states is not a parity check, since one-step bf16 differences of the projections
(float32 against float64 accumulation) grow through the layers.
"""

import numpy as np
import pytest
import torch

import oracle
from synth import layer_inputs

pytestmark = pytest.mark.gpu

THETA = 500000.0

CASES = {
    "d64-g2-b2-3layers": dict(B=2, Hq=4, Hkv=2, d=64, L=1024, b=256, P=128, anchor=0, layers=3),
    "d128-g4-a256-2layers": dict(B=1, Hq=8, Hkv=2, d=128, L=1024, b=512, P=256, anchor=256, layers=2),
}


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def H():
    from tests import harness
    return harness


@pytest.mark.parametrize("name", list(CASES))
def test_encode_layers_matches_oracle(name):
    import block_sparse_attention_star_b200 as star

    c = CASES[name]
    B, Hq, Hkv, d, L, b, nl = c["B"], c["Hq"], c["Hkv"], c["d"], c["L"], c["b"], c["layers"]
    hidden = Hq * d
    dev = torch.device("cuda", 0)
    x0, ws = layer_inputs(5, nl, B, L, hidden, Hq * d, Hkv * d, device=dev)
    ws32 = [tuple(w.float() for w in layer) for layer in ws]
    shape = star.StarShape.make(B=B, Hq=Hq, Hkv=Hkv, d=d, L=L, b=b, T_max=16, page_tokens=c["P"],
                                anchor=c["anchor"])
    caches = [star.PagedKVCache(shape, device=dev) for _ in range(nl)]
    pos = torch.arange(L, dtype=torch.int32, device=dev).repeat(B, 1).contiguous()
    x = x0.clone()
    q = torch.empty((B, L, Hq, d), dtype=torch.bfloat16, device=dev)
    k = torch.empty((B, L, Hkv, d), dtype=torch.bfloat16, device=dev)
    v = torch.empty_like(k)
    o = torch.empty_like(q)
    seen = []  # per layer: (q, k, v, o) as the library read and wrote them

    def model(layer, stage, x, q, k, v, o):
        wq, wk, wv, wo = ws32[layer]
        xf = x.view(B * L, hidden).float()
        if stage == star.STAR_LAYER_QKV:
            q.copy_((xf @ wq).view(q.shape).to(torch.bfloat16))
            k.copy_((xf @ wk).view(k.shape).to(torch.bfloat16))
            v.copy_((xf @ wv).view(v.shape).to(torch.bfloat16))
            seen.append([q.clone(), k.clone(), v.clone()])
        else:
            seen[layer].append(o.clone())
            x.copy_((xf + o.view(B * L, Hq * d).float() @ wo).view(x.shape).to(torch.bfloat16))

    star.star_encode_layers(shape, caches, pos, x, q, k, v, o, model)
    torch.cuda.synchronize()
    assert star.star_device_status() == 0
    assert len(seen) == nl and all(len(s) == 4 for s in seen)

    h = H()
    for li, (ql, kl, vl, ol) in enumerate(seen):
        for bi in range(B):
            o_ref, ck, cv = oracle.phase1(h.to64(ql[bi]), h.to64(kl[bi]), h.to64(vl[bi]), np.arange(L), b, THETA,
                                          c["anchor"] or None)
            h.assert_out(ol[bi], o_ref, f"layer {li} attention output (seq {bi})")
            kg, vg = caches[li].gather(bi, 0, L)
            diff = np.abs(h.to64(kg) - ck)
            assert np.all(diff <= np.abs(ck) * 2.0 ** -7) and np.count_nonzero(diff) <= 4, f"layer {li} cache K"
            assert np.array_equal(h.to64(vg), cv), f"layer {li} cache V (seq {bi})"
    # the layers really chained: the last layer's inputs came from the updated hidden states
    assert not torch.equal(seen[0][0], seen[-1][0])


def test_encode_layers_stops_on_a_callback_error():
    import block_sparse_attention_star_b200 as star

    dev = torch.device("cuda", 0)
    shape = star.StarShape.make(B=1, Hq=4, Hkv=2, d=64, L=512, b=256, T_max=16)
    caches = [star.PagedKVCache(shape, device=dev) for _ in range(2)]
    pos = torch.arange(512, dtype=torch.int32, device=dev).view(1, -1).contiguous()
    x = torch.zeros((1, 512, 256), dtype=torch.bfloat16, device=dev)
    q = torch.zeros((1, 512, 4, 64), dtype=torch.bfloat16, device=dev)
    k = torch.zeros((1, 512, 2, 64), dtype=torch.bfloat16, device=dev)
    calls = []

    def model(layer, stage, *_):
        calls.append((layer, stage))
        if layer == 1:
            raise ValueError("caller's model failed")

    with pytest.raises(ValueError):
        star.star_encode_layers(shape, caches, pos, x, q, k, k.clone(), q.clone(), model)
    assert calls == [(0, star.STAR_LAYER_QKV), (0, star.STAR_LAYER_OUT), (1, star.STAR_LAYER_QKV)]
    torch.cuda.synchronize()
    assert star.star_device_status() == 0
