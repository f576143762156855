"""The N > 1 host logic of bench.py on CPU with world_size-2 gloo ranks.

Each rank runs an independent sequence batch (its own seed, no collective on the
data path); the job's time is the slowest rank's; the reported value counts the
context tokens of all ranks.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        wl = bench.rank_workload("llama8b-32k", rank)
        slowest = bench.max_over_ranks(100.0 + 7.0 * rank, torch.device("cpu"))
        from synth import make_inputs
        tiny = bench.rank_workload("tiny", rank)
        x = make_inputs(tiny, "cpu", parts=("query",))["q_query"].float().sum().item()
        q.put((rank, wl.seed, slowest, bench.job_value(world, wl.context_tokens(), slowest), x))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_sequences_and_take_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    seeds = [r[1] for r in res]
    assert seeds == [0, 1]                          # independent sequences per rank
    assert all(r[2] == 107.0 for r in res)          # max over ranks
    assert all(r[3] == pytest.approx(2 * 32768 / 0.107) for r in res)
    assert res[0][4] != res[1][4]                   # different data on each rank
