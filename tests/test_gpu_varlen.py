"""GPU parity for ragged last blocks and batches of variable-length sequences.

star_shape.seq_len gives each sequence its own context length L_s <= L (the
capacity); its last block holds L_s - (n_s-1) b tokens, its query and generated
tokens follow L_s, and the partials of blocks it does not have are empty
(O = 0, LSE = -inf) and skipped by the merge.  Compared element by element with the
oracle (same tolerances as the main parity tests; rows past L_s are padding and
not compared), plus: Phase-1 outputs of a batch equal each sequence run alone, bit
for bit.
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
    "d128-g4-var": Workload("d128-g4-var", B=3, Hq=8, Hkv=2, d=128, L=2048, b=512, T=40, S=3, peaky=True,
                            seq_lens=(2048, 1700, 612)),
    "d64-g2-var-p128": Workload("d64-g2-var-p128", B=2, Hq=4, Hkv=2, d=64, L=1024, b=256, T=7, S=2, peaky=False,
                                page_tokens=128, seq_lens=(1000, 256)),
    "tiny-ragged": dataclasses.replace(get_config("tiny"), name="tiny-ragged", seq_lens=(777,)),
    "d128-g8-var-t130": Workload("d128-g8-var-t130", B=2, Hq=16, Hkv=2, d=128, L=1024, b=256, T=130, S=2,
                                 peaky=True, seq_lens=(1024, 333)),
    # six sequences, the shortest first and a one-token context: per-sequence item tables
    # and chunk counts in the decode (one chunk for the first sequence, four for the third)
    "d64-g4-var-b6": Workload("d64-g4-var-b6", B=6, Hq=8, Hkv=2, d=64, L=1024, b=256, T=9, S=2, peaky=True,
                              seq_lens=(1, 130, 1024, 257, 640, 999)),
}


def _check_all(wl, res, inp, ref):
    h = H()
    for bi in range(wl.B):
        Ls = wl.ctx_len(bi)
        h.assert_out(res["o_ctx"][bi][:Ls], ref["o_ctx"][bi][:Ls], f"phase1 rows (seq {bi}, L_s {Ls})")
        k, v = res["cache"].gather(bi, 0, Ls + wl.T + wl.S)
        ck = ref["cache_k"][bi]
        kg = h.to64(k[:Ls])
        diff = np.abs(kg - ck)
        assert np.all(diff <= np.abs(ck) * 2.0 ** -7) and np.count_nonzero(diff) <= 4, f"cache K (seq {bi})"
        assert np.array_equal(h.to64(v[:Ls]), ref["cache_v"][bi]), f"cache V (seq {bi})"
    h.assert_out(res["o_part"], ref["o_part"], "phase2 partial O")
    h.assert_lse(res["lse_part"], ref["lse_part"], "phase2 partial LSE")
    h.assert_out(res["o_query"], ref["o_query"], "merged query O")
    h.assert_lse(res["lse_query"], ref["lse_query"], "merged query LSE")
    h.assert_out(res["o_dec"][:, :, 0], ref["o_dec"], "decode O")
    h.assert_lse(res["lse_dec"], ref["lse_dec"], "decode LSE")


@pytest.mark.parametrize("name", list(SMALL))
def test_varlen_batch_matches_oracle(name):
    wl = SMALL[name]
    h = H()
    inp = make_inputs(wl, "cuda")
    res = h.run_gpu(wl, inp)
    assert res["status"] == 0
    ref = oracle.run_star(h.oracle_inputs(inp), wl.L, wl.b, wl.theta)
    _check_all(wl, res, inp, ref)
    # partials of blocks a sequence does not have are empty
    n = -(-wl.L // wl.b)
    for bi in range(wl.B):
        n_s = -(-wl.ctx_len(bi) // wl.b)
        assert torch.all(res["lse_part"][n_s:n, bi] == -float("inf"))
        assert torch.all(res["o_part"][n_s:n, bi] == 0)


def test_phase1_of_a_batch_equals_each_sequence_alone():
    import block_sparse_attention_star_b200 as star
    h = H()
    wl = SMALL["d128-g4-var"]
    inp = make_inputs(wl, "cuda", parts=("ctx",))
    res = h.run_gpu(wl, inp, phases=("phase1",))
    for bi in range(wl.B):
        one = dataclasses.replace(wl, B=1, seq_lens=(wl.ctx_len(bi),))
        inp1 = {k: v[bi:bi + 1].contiguous() for k, v in inp.items() if k != "seq_len"}
        r1 = h.run_gpu(one, inp1, phases=("phase1",))
        Ls = wl.ctx_len(bi)
        assert torch.equal(res["o_ctx"][bi][:Ls], r1["o_ctx"][0][:Ls]), f"seq {bi}"
    assert star.star_device_status() == 0


def test_varlen_rejects_positions_inside_the_context():
    import block_sparse_attention_star_b200 as star
    h = H()
    wl = SMALL["d64-g2-var-p128"]
    shape = h.shape_of(wl)
    cache = star.PagedKVCache(shape)
    kv = torch.zeros((wl.B, 1, wl.Hkv, wl.d), dtype=torch.bfloat16, device="cuda")
    pos = torch.zeros((wl.B, 1), dtype=torch.int32, device="cuda")
    with pytest.raises(star.StarError) as e:
        star.star_kv_append(shape, cache, kv, kv, pos, wl.L - 1, 1)
    assert e.value.code == star.STAR_ERR_INVALID_ARG


def test_llama70b_shape_with_a_ragged_sequence_sampled():
    """B = 2 at the 70B shape: one full 128K context and one of 100000 tokens (6 blocks of
    16384 and a ragged seventh of 1696)."""
    h = H()
    wl = dataclasses.replace(get_config("llama70b-128k"), name="llama70b-128k-var", seq_lens=(131072, 100000))
    inp = make_inputs(wl, "cuda")
    res = h.run_gpu(wl, inp)
    assert res["status"] == 0
    theta = wl.theta
    for bi in range(wl.B):
        Ls = wl.ctx_len(bi)
        k = h.to64(inp["k_ctx"][bi][:Ls])
        v = h.to64(inp["v_ctx"][bi][:Ls])
        pos = inp["pos_ctx"][bi][:Ls].cpu().numpy().astype(np.int64)
        rows = np.unique(np.concatenate([h.sample_rows(dataclasses.replace(wl, L=Ls - Ls % wl.b), 4),
                                         [Ls - 1, Ls - 129, (Ls - 1) // wl.b * wl.b]]))
        rows = rows[rows < Ls]
        ref_rows = oracle.phase1_rows(rows, h.to64(inp["q_ctx"][bi][torch.from_numpy(rows).cuda()]), k, v, pos,
                                      wl.b, theta)
        h.assert_out(res["o_ctx"][bi][torch.from_numpy(rows).cuda()], ref_rows, f"phase1 sampled rows (seq {bi})")
        ck = oracle.rope_bf16(k, pos, theta)
        qpos = inp["pos_query"][bi].cpu().numpy().astype(np.int64)
        ck, cv = oracle.append_tail(ck, v, h.to64(inp["k_query"][bi]), h.to64(inp["v_query"][bi]), qpos, theta)
        n_parts = -(-wl.L // wl.b)
        Op, Lp = oracle.phase2_partials(h.to64(inp["q_query"][bi]), qpos, ck, cv, Ls, wl.b, theta, n_parts)
        Oq, Lq = oracle.lse_merge(Op, Lp)
        h.assert_out(res["o_part"][:, bi], Op, "phase2 partial O")
        h.assert_lse(res["lse_part"][:, bi], Lp, "phase2 partial LSE")
        h.assert_out(res["o_query"][bi], Oq, "merged O")
        h.assert_lse(res["lse_query"][bi], Lq, "merged LSE")
        for s in range(wl.S):
            kd, vd = h.to64(inp["k_dec"][s, bi]), h.to64(inp["v_dec"][s, bi])
            p = int(inp["pos_dec"][s, bi])
            if s in (0, wl.S - 1):
                O, LSE, ck, cv = oracle.decode_step(h.to64(inp["q_dec"][s, bi]), kd, vd, p, ck, cv, theta)
                h.assert_out(res["o_dec"][s, bi], O, f"decode step {s} O")
                h.assert_lse(res["lse_dec"][s, bi], LSE[0], f"decode step {s} LSE")
            else:
                ck, cv = oracle.append_tail(ck, cv, kd, vd, [p], theta)
