"""The multi-GPU star exchange (block_sparse_attention_star_b200.shard) on CPU with gloo ranks.

Each rank owns a contiguous block range (``block_range``) of one sequence, computes the
per-block partials of the query rows and of every decode token over its own keys only
(here with the oracle, on the CPU: the rank's blocks of ``oracle.phase2_partials``, and
``oracle.attend`` over the rank's keys for decode), exchanges them through
``ShardExchange.gather_merge`` (padded all-gathers over gloo), and merges them with
``oracle.lse_merge``.  The merged result must equal the oracle's merge over all blocks,
and brute-force attention over the whole cache ("组装全局结果": the merge is exact).
World sizes 2 and 3, with block counts that do and do not divide evenly (padding with
empty partials).  The partials travel as float32, as on the GPU, so the comparisons allow
float32 rounding (a missing, duplicated or misplaced partial is off by far more).
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_attention_star_b200.shard import block_range


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_block_ranges_are_contiguous_and_balanced():
    for n in range(1, 20):
        for world in range(1, n + 1):
            ranges = [block_range(n, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [e - b for b, e in ranges]
            assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        block_range(2, 3, 0)


def _problem(L, b, T, S, seed=80):
    import oracle
    rng = np.random.default_rng(seed)
    f = lambda *sh: oracle.round_to_bf16(rng.standard_normal(sh))
    Hq, Hkv, d, theta = 4, 2, 16, 500000.0
    k, v = f(L, Hkv, d) * 2, f(L, Hkv, d)
    qq, kq, vq = f(T, Hq, d), f(T, Hkv, d), f(T, Hkv, d)
    qd, kd, vd = f(S, 1, Hq, d), f(S, 1, Hkv, d), f(S, 1, Hkv, d)
    ck = oracle.rope_bf16(k, np.arange(L), theta)
    ck, cv = oracle.append_tail(ck, v, kq, vq, L + np.arange(T), theta)
    return dict(L=L, b=b, T=T, S=S, theta=theta, ck=ck, cv=cv, qq=qq, qd=qd, kd=kd, vd=vd)


def _worker(rank, world, port, L, b, q_out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from block_sparse_attention_star_b200.shard import ShardExchange

        def merge(o_all, lse_all):
            O, LSE = oracle.lse_merge(o_all.numpy().astype(np.float64), lse_all.numpy().astype(np.float64))
            return O, LSE

        P = _problem(L, b, T=3, S=2)
        n = -(-L // b)
        ex = ShardExchange(n, device="cpu", merge_fn=merge)
        i0, i1 = ex.begin, ex.end
        theta = P["theta"]
        # Query rows: this rank's blocks of the per-block partials (the tail in the last block).
        Op, Lp = oracle.phase2_partials(P["qq"], L + np.arange(P["T"]), P["ck"], P["cv"], L, b, theta)
        mine_o = torch.from_numpy(Op[i0:i1].reshape(i1 - i0, -1, Op.shape[-1]))
        mine_l = torch.from_numpy(Lp[i0:i1].reshape(i1 - i0, -1))
        Oq, Lq = ex.gather_merge(mine_o, mine_l)
        # Decode: each step appends its token on the last rank; every rank attends with its keys.
        ck, cv = P["ck"], P["cv"]
        dec = []
        for s in range(P["S"]):
            pos = L + P["T"] + s
            ck, cv = oracle.append_tail(ck, cv, P["kd"][s], P["vd"][s], [pos], theta)
            qr = oracle.rope_bf16(P["qd"][s], [pos], theta)
            hi = ck.shape[0] if i1 == n else i1 * b
            O, LSE = oracle.attend(qr, ck[i0 * b:hi], cv[i0 * b:hi])
            Od, Ld = ex.gather_merge(torch.from_numpy(O.reshape(1, -1, O.shape[-1])),
                                     torch.from_numpy(LSE.reshape(1, -1)), slots=1)
            dec.append((Od, Ld))
        q_out.put((rank, (i0, i1), Oq, Lq, dec))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,L,b", [(2, 64, 16), (2, 80, 16), (3, 64, 16)])
def test_sharded_partials_exchange_and_merge_equal_the_whole_context(world, L, b):
    import oracle
    from tests.test_oracle_pins import lse_lib, sdpa
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, L, b, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    got.sort(key=lambda x: x[0])
    n = -(-L // b)
    assert [g[1] for g in got] == [block_range(n, world, r) for r in range(world)]
    P = _problem(L, b, T=3, S=2)
    theta = P["theta"]
    Op, Lp = oracle.phase2_partials(P["qq"], L + np.arange(P["T"]), P["ck"], P["cv"], L, b, theta)
    Oq, Lq = oracle.lse_merge(Op, Lp)
    qr = oracle.rope_bf16(P["qq"], L + np.arange(P["T"]), theta)
    mask = np.arange(P["ck"].shape[0])[None, :] <= (L + np.arange(P["T"]))[:, None]
    tol = dict(rtol=1e-6, atol=1e-6)
    for rank, _, O, LSE, dec in got:
        # every rank ends with the same global result
        np.testing.assert_allclose(O.reshape(Oq.shape), Oq, **tol)
        np.testing.assert_allclose(LSE.reshape(Lq.shape), Lq, **tol)
        np.testing.assert_allclose(O.reshape(Oq.shape), sdpa(qr, P["ck"], P["cv"], mask), **tol)
        np.testing.assert_allclose(LSE.reshape(Lq.shape), lse_lib(qr, P["ck"], mask), **tol)
        ck, cv = P["ck"], P["cv"]
        for s in range(P["S"]):
            Od_ref, Ld_ref, ck, cv = oracle.decode_step(P["qd"][s], P["kd"][s], P["vd"][s], L + P["T"] + s, ck, cv,
                                                        theta)
            Od, Ld = dec[s]
            np.testing.assert_allclose(Od.reshape(Od_ref.shape), Od_ref, **tol)
            np.testing.assert_allclose(Ld.reshape(Ld_ref.shape), Ld_ref, **tol)
