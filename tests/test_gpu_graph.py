"""The whole hot path captured in a CUDA graph and replayed.

Every entry point of one step (Phase 1, Phase 2 with its query append, the merge and
the decode steps with their appends) is a sequence of kernel launches on the caller's
stream with no allocation and no host synchronisation, so it can be captured once a
first call has set up each kernel (shared-memory opt-ins).  A replay recomputes the
step from the same inputs: every output must be bit-identical to the eager run, and
two replays to each other (context anchors at caller ids and per-sequence lengths
included).
"""

import dataclasses

import pytest
import torch

from synth import Workload, get_config

pytestmark = pytest.mark.gpu

OUTS = ["o_ctx", "o_q", "lse_q", "o_dec", "lse_dec"]


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _outputs(run):
    return {n: getattr(run, n).clone() for n in OUTS}


def _poison(run):
    # the same sentinel before the eager step and before each replay, so that rows no
    # step writes (past a shorter sequence's context) compare equal
    for n in OUTS:
        getattr(run, n).fill_(-7.0)


@pytest.mark.parametrize("wl", [
    get_config("tiny"),
    Workload("d128-g4-b2-graph", B=2, Hq=8, Hkv=2, d=128, L=2048, b=512, T=40, S=5, peaky=True),
    dataclasses.replace(get_config("llama8b-32k"), S=4),
    Workload("graph-anchor-offset", B=1, Hq=8, Hkv=2, d=128, L=2048, b=512, T=16, S=3, peaky=False,
             anchor=256, anchor_ids="offset"),
    Workload("graph-varlen", B=3, Hq=8, Hkv=2, d=128, L=2048, b=512, T=16, S=3, peaky=True,
             seq_lens=(2048, 1500, 700)),
], ids=lambda w: w.name)
def test_step_replays_bit_identically(wl):
    import block_sparse_attention_star_b200 as star
    from bench import StarRun

    dev = torch.device("cuda", 0)
    run = StarRun(wl, dev)
    _poison(run)
    run.step()  # eager: sets up every kernel before capture
    torch.cuda.synchronize()
    assert star.star_device_status() == 0
    eager = _outputs(run)

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run.step()
    for rep in range(2):
        _poison(run)
        graph.replay()
        torch.cuda.synchronize()
        assert star.star_device_status() == 0
        got = _outputs(run)
        for n in OUTS:
            assert torch.equal(got[n], eager[n]), f"{wl.name}: replay {rep} changed {n}"
    del graph
