#!/usr/bin/env python
"""Benchmark of the Star Attention hot path on NVIDIA B200.

One step = the whole hot path over one batch of the workload, through the C ABI:
RoPE + KV append and Phase-1 anchor-augmented attention (star_phase1_encode),
query append + per-block partials (star_phase2_partial), the exact merge
(star_lse_merge), and S decode steps (star_decode_step).  Inputs are seeded
synthetic tensors already resident in HBM when the timed region starts; the
`e2e` leg repeats the step from pinned host buffers with the copies inside the
timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl star|reference]
    python bench.py --layers N [--config NAME]   # N layers of context encoding (star_encode_layers)

Multi-GPU (torchrun): every rank runs its own independent sequence batch (the
path partitions by sequence; no collective on the data path); time is the max
over ranks.  `--impl reference` times the CPU oracle (float64 numpy) on bounded
samples of the same workload's step on the host cores and reports the whole step
extrapolated from them (same metric and unit); `--oracle-full` times the whole
oracle on a small workload.
"""

from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import threading
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import get_config, make_inputs  # noqa: E402

METRIC = "Phase-1 ctx tok/s (% BF16 peak) at 128K; Phase-2 decode µs/step (HBM GB/s)"
# Datasheet figures for one B200, for the nominal fractions beside the measured ones: dense bf16
# tensor throughput (NVIDIA's 2:4-sparse figure halved) and HBM3e bandwidth (about 8 TB/s).
NOMINAL = {"bf16_tflops": 2250.0, "hbm_gbs": 8000.0}
UNIT = "ctx tok/s"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="llama8b-128k-b32768")
    ap.add_argument("--impl", default="star", choices=["star", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=8, help="Phase-1 rows per block in the oracle sample")
    ap.add_argument("--oracle-full", action="store_true",
                    help="time the whole CPU oracle on the full workload (small workloads only) and exit")
    ap.add_argument("--shard", action="store_true",
                    help="multi-GPU Star Attention: every rank owns a block range of the same sequences "
                         "(Phase 1 on its blocks, Phase-2 and decode partials exchanged and merged)")
    ap.add_argument("--exchange", default="p2p", choices=["p2p", "nccl"],
                    help="--shard: partials all-gathered by NCCL, or pushed by the kernels into every GPU's "
                         "exchange buffer over peer memory")
    ap.add_argument("--layers", type=int, default=0,
                    help="time N layers of context encoding (star_encode_layers, random projections) instead")
    return ap.parse_args()


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return {"hbm_gbs": pk["hbm_gbs"], "bf16": pk["bf16_tflops"], "bf16_sustained": pk["bf16_tflops_sustained"],
                "kind": "of measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "kind": "of fallback"}


# ---------------------------------------------------------------------------
# Clock sampling during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            target = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            target = str(device_index)
        self.cmd = ["nvidia-smi", "-i", target, "--query-gpu=" + ",".join(self.FIELDS),
                    "--format=csv,noheader,nounits", "-lms", "50"]

    def __enter__(self):
        """Start nvidia-smi and return once it has produced its first sample, so that the timed
        region that follows is covered from its start."""
        self.samples = []
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return self

        def read():
            for ln in self.proc.stdout:
                if ln.strip():
                    self.samples.append((time.monotonic(), ln))

        self.reader = threading.Thread(target=read, daemon=True)
        self.reader.start()
        deadline = time.monotonic() + 5.0
        while not self.samples and time.monotonic() < deadline:
            time.sleep(0.01)
        self.t0 = time.monotonic()
        return self

    def __exit__(self, *exc):
        t1 = time.monotonic()
        if self.proc is not None:
            time.sleep(0.06)  # the sample that closes the window
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.reader.join(timeout=5)
            inside = [ln for t, ln in self.samples if self.t0 <= t <= t1 + 0.06]
            after = [ln for t, ln in self.samples if t >= self.t0]
            self.lines = inside or after[:1]

    def summary(self):
        sm, smax, reasons = [], [], set()
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < len(self.FIELDS):
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# The CUDA path
# ---------------------------------------------------------------------------
def launches_per_step(star, shape, wl, anchor_ids: bool) -> int:
    """Library kernel launches in one step.  Phase 1: RoPE + KV append, tail zero-fill,
    RoPE(Q), attention (+ the anchor keys at caller ids).  Phase 2: query KV append,
    RoPE(Q), attention (+ the chunk merge when blocks are split into chunks, i.e. when
    the workspace holds more than RoPE(Q)).  The query merge.  Per decode step: the
    decode kernel (one launch: its chunking keeps the items within one launch) and its
    merge."""
    q_bytes = -(-wl.B * wl.T * wl.Hq * wl.d * 2 // 256) * 256
    chunked = star.star_workspace_size(shape, star.STAR_OP_PHASE2, wl.T) > q_bytes
    return (4 + (1 if anchor_ids else 0)) + (3 + (1 if chunked else 0)) + 1 + 2 * wl.S


def workload_config(wl, world):
    """The `config` object of the JSON line (the same for both arms)."""
    return {"workload": wl.name, "B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv, "d": wl.d, "L": wl.L, "b": wl.b,
            "n": wl.n, "T": wl.T, "S": wl.S, "page_tokens": wl.page_tokens, "anchor": wl.a,
            "anchor_ids": wl.anchor_ids, "seq_lens": list(wl.seq_lens) if wl.seq_lens else None,
            "parallelism": f"independent sequences per GPU x{world}",
            "l2": "inputs larger than L2 (no flush)"}


def workload_shape(wl):
    """The C-ABI shape of a workload: sizes, anchor and per-sequence context lengths."""
    import block_sparse_attention_star_b200 as star
    return star.StarShape.make(B=wl.B, Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d, L=wl.L, b=wl.b, T_max=wl.T_max,
                               page_tokens=wl.page_tokens, rope_theta=wl.theta, anchor=wl.anchor,
                               seq_len=wl.seq_lens)


class StarRun:
    """Buffers and the step sequence of one workload on one GPU."""

    def __init__(self, wl, device):
        import block_sparse_attention_star_b200 as star
        self.star, self.wl, self.dev = star, wl, device
        self.inp = make_inputs(wl, device)
        self.shape = workload_shape(wl)
        self.cache = star.PagedKVCache(self.shape, device=device)
        self.o_ctx = torch.empty_like(self.inp["q_ctx"])
        self.o_part, self.lse_part = star.alloc_partials(self.shape, wl.T, device)
        self.ws2 = star.workspace(self.shape, star.STAR_OP_PHASE2, wl.T, device)
        self.wsd = star.workspace(self.shape, star.STAR_OP_DECODE, 0, device)
        self.ws1 = (star.workspace(self.shape, star.STAR_OP_PHASE1_ANCHOR, 0, device)
                    if "anchor_pos" in self.inp else None)
        self.o_q = torch.empty((wl.B, wl.T, wl.Hq, wl.d), dtype=torch.bfloat16, device=device)
        self.lse_q = torch.empty((wl.B, wl.T, wl.Hq), dtype=torch.float32, device=device)
        self.o_dec = torch.empty((wl.S, wl.B, 1, wl.Hq, wl.d), dtype=torch.bfloat16, device=device)
        self.lse_dec = torch.empty((wl.S, wl.B, wl.Hq), dtype=torch.float32, device=device)
        self.launches_per_step = launches_per_step(star, self.shape, wl, anchor_ids="anchor_pos" in self.inp)

    def step(self, ev=None):
        """One pass of the hot path.  ev: optional dict of (start, stop) event lists to record."""
        s, wl, inp = self.star, self.wl, self.inp
        if ev and "p1" in ev:
            s.star_set_trace_events(*ev["p1"])
        if self.ws1 is not None:
            s.star_phase1_encode_anchored(self.shape, self.cache, inp["q_ctx"], inp["k_ctx"], inp["v_ctx"],
                                          inp["pos_ctx"], inp["anchor_pos"], self.o_ctx, self.ws1)
        else:
            s.star_phase1_encode(self.shape, self.cache, inp["q_ctx"], inp["k_ctx"], inp["v_ctx"], inp["pos_ctx"],
                                 self.o_ctx)
        if ev and "p2" in ev:
            s.star_set_trace_events(*ev["p2"])
        s.star_phase2_partial(self.shape, self.cache, inp["q_query"], inp["k_query"], inp["v_query"], inp["pos_query"],
                              wl.T, self.o_part, self.lse_part, self.ws2)
        if ev:
            s.star_set_trace_events(None, None)
        if ev and "merge" in ev:
            ev["merge"][0].record()
        s.star_lse_merge(self.shape.n, wl.B * wl.T * wl.Hq, wl.d, self.o_part, self.lse_part, self.o_q, self.lse_q)
        if ev and "merge" in ev:
            ev["merge"][1].record()
        # ev["dec_span"] brackets the S decode steps with nothing between their launches;
        # ev["dec"] (a separate instrumented step) brackets every decode attention kernel.
        if ev and "dec_span" in ev:
            ev["dec_span"][0].record()
        for st in range(wl.S):
            if ev and "dec" in ev:
                s.star_set_trace_events(*ev["dec"][st])
            s.star_decode_step(self.shape, self.cache, inp["q_dec"][st], inp["k_dec"][st], inp["v_dec"][st],
                               inp["pos_dec"][st], wl.L + wl.T + st, self.o_dec[st], self.lse_dec[st], self.wsd)
        if ev and "dec_span" in ev:
            ev["dec_span"][1].record()
        if ev:
            s.star_set_trace_events(None, None)


class ShardRun:
    """One rank's share of a workload when the context's blocks are sharded over the ranks:
    its block range of every sequence (the same sequences on every rank), the anchor's
    tokens when the range does not hold block 1, and the tail on the rank with the last block."""

    def __init__(self, wl, device, exchange="p2p"):
        import block_sparse_attention_star_b200 as star
        from block_sparse_attention_star_b200.shard import PeerExchange, ShardExchange
        self.star, self.wl, self.dev = star, wl, device
        inp = make_inputs(wl, device)
        self.shape = workload_shape(wl)
        self.ex = ShardExchange(wl.n, device=device)
        i0, i1 = self.ex.begin, self.ex.end
        self.tail = i1 == wl.n
        sl = slice(i0 * wl.b, i1 * wl.b)
        a = wl.a
        self.ctx = {x: inp[x][:, sl].contiguous() for x in ("q_ctx", "k_ctx", "v_ctx", "pos_ctx")}
        self.anchor = {x: inp[x][:, :a].contiguous() for x in ("k_ctx", "v_ctx", "pos_ctx")}
        self.query = {x: inp[x] for x in ("q_query", "k_query", "v_query", "pos_query")}
        self.dec = {x: inp[x] for x in ("q_dec", "k_dec", "v_dec", "pos_dec")}
        del inp
        self.cache = star.PagedKVCache(self.shape, device=device)
        self.o_ctx = torch.empty_like(self.ctx["q_ctx"])
        nl = i1 - i0
        self.o_part = torch.empty((nl, wl.B, wl.T, wl.Hq, wl.d), dtype=torch.float32, device=device)
        self.lse_part = torch.empty((nl, wl.B, wl.T, wl.Hq), dtype=torch.float32, device=device)
        self.ws2 = star.workspace(self.shape, star.STAR_OP_PHASE2, wl.T, device)
        self.wsd = star.workspace(self.shape, star.STAR_OP_DECODE, 0, device)
        self.o_q = torch.empty((wl.B, wl.T, wl.Hq, wl.d), dtype=torch.bfloat16, device=device)
        self.lse_q = torch.empty((wl.B, wl.T, wl.Hq), dtype=torch.float32, device=device)
        self.po = torch.empty((1, wl.B, wl.Hq, wl.d), dtype=torch.float32, device=device)
        self.pl = torch.empty((1, wl.B, wl.Hq), dtype=torch.float32, device=device)
        self.o_dec = torch.empty((wl.S, wl.B, wl.Hq, wl.d), dtype=torch.bfloat16, device=device)
        self.lse_dec = torch.empty((wl.S, wl.B, wl.Hq), dtype=torch.float32, device=device)
        self.p2p = exchange == "p2p"
        if self.p2p:
            self.pq = PeerExchange(wl.B * wl.T * wl.Hq, wl.d, self.ex.nmax, device=device)
            self.pd = PeerExchange(wl.B * wl.Hq, wl.d, 1, device=device)
            self.ws2p = star.workspace(self.shape, star.STAR_OP_PHASE2_PUSH, wl.T, device)

    def launches_per_step(self) -> int:
        """Library kernel launches of one step on this rank.  Phase 1: RoPE + KV append of the
        range, of the anchor (a range after block 1), the tail zero-fill (the last range),
        RoPE(Q), attention.  Phase 2: the query's KV append (last range), RoPE(Q), attention,
        the chunk merge (when blocks are split into chunks), the exchange's merge.  Per decode
        step: the decode kernel, its chunk merge, the exchange's merge."""
        wl, star = self.wl, self.star
        q_bytes = -(-wl.B * wl.T * wl.Hq * wl.d * 2 // 256) * 256
        chunked = star.star_workspace_size(self.shape, star.STAR_OP_PHASE2, wl.T) > q_bytes
        p1 = 3 + (1 if self.ex.begin > 0 else 0) + (1 if self.tail else 0)
        if self.p2p:  # attention + push (merge-scatter) + the exchange merge; decode: kernel, push, merge
            return p1 + 2 + (1 if self.tail else 0) + 2 + 3 * wl.S
        p2 = 2 + (1 if self.tail else 0) + (1 if chunked else 0) + 1
        return p1 + p2 + 3 * wl.S

    def step(self):
        s, wl, c, sh = self.star, self.wl, self.ctx, self.ex.shard()
        s.star_phase1_encode_shard(self.shape, self.cache, sh, c["q_ctx"], c["k_ctx"], c["v_ctx"], c["pos_ctx"],
                                   self.anchor["k_ctx"], self.anchor["v_ctx"], self.anchor["pos_ctx"], self.o_ctx)
        q = self.query
        d = self.dec
        if self.p2p:
            # The kernels push every partial into each GPU's exchange buffer; each GPU merges its own.
            s.star_phase2_partial_shard_push(self.shape, self.cache, sh, q["q_query"],
                                             q["k_query"] if self.tail else None, q["v_query"] if self.tail else None,
                                             q["pos_query"], wl.T, self.pq.ex, self.pq.next_epoch(), self.ws2p)
            self.pq.merge(self.o_q, self.lse_q)
            for st in range(wl.S):
                s.star_decode_partial_shard_push(self.shape, self.cache, sh, d["q_dec"][st], d["k_dec"][st],
                                                 d["v_dec"][st], d["pos_dec"][st], wl.L + wl.T + st, self.pd.ex,
                                                 self.pd.next_epoch(), self.wsd)
                self.pd.merge(self.o_dec[st], self.lse_dec[st])
            return
        s.star_phase2_partial_shard(self.shape, self.cache, sh, q["q_query"], q["k_query"] if self.tail else None,
                                    q["v_query"] if self.tail else None, q["pos_query"], wl.T, self.o_part,
                                    self.lse_part, self.ws2)
        rows = wl.B * wl.T * wl.Hq
        self.ex.gather_merge(self.o_part.view(-1, rows, wl.d), self.lse_part.view(-1, rows), self.o_q, self.lse_q)
        for st in range(wl.S):
            s.star_decode_partial_shard(self.shape, self.cache, sh, d["q_dec"][st], d["k_dec"][st], d["v_dec"][st],
                                        d["pos_dec"][st], wl.L + wl.T + st, self.po[0], self.pl[0], self.wsd)
            self.ex.gather_merge(self.po.view(1, -1, wl.d), self.pl.view(1, -1), self.o_dec[st], self.lse_dec[st],
                                 slots=1)


def run_shard(args, rank, world, local_rank):
    """Blocks sharded over the ranks: the whole job processes one batch of sequences per step
    (strong scaling: the total work is fixed as the rank count grows)."""
    import torch.distributed as dist
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = get_config(args.config)
    run = ShardRun(wl, dev, args.exchange)
    for _ in range(max(3, args.warmup)):
        run.step()
    torch.cuda.synchronize()
    if run.star.star_device_status() != 0:
        raise RuntimeError("device error after warm-up")
    K = args.steps
    t0, t1 = _ev(), _ev()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        t0.record()
        for _ in range(K):
            run.step()
        t1.record()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    status = run.star.star_device_status()
    ms_step = max_over_ranks(t0.elapsed_time(t1), dev) / K
    if rank == 0:
        nl = run.ex.n_local
        line = {
            "metric": METRIC, "value": wl.context_tokens() / (ms_step * 1e-3), "unit": UNIT, "n_gpus": world,
            "steps": K, "warmup": max(3, args.warmup), "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16; 1% of context key rows x8 where the workload says peaky)",
            "config": dict(workload_config(wl, world), parallelism=f"context blocks sharded over {world} GPUs"),
            "exchange": (f"per query call and per decode step: the partial kernels push the f32 (O, LSE) "
                         f"partials into every GPU's exchange buffer over peer memory; each GPU merges its own "
                         f"(rank 0 holds {nl} of {wl.n} blocks)") if run.p2p else
                        (f"per query call and per decode step: all-gather of the f32 (O, LSE) partials "
                         f"(rank 0 holds {nl} of {wl.n} blocks), then star_lse_merge on every rank"),
            "gpu_launches": run.launches_per_step() * K,
            "device_status": status, "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)


def measured_traffic(B: int, L: int):
    """DRAM bytes of one Phase-1 launch from the committed ncu record, scaled by context tokens;
    None when the kernel sources changed since the counters were taken."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "attn_phase1_traffic.json")) as f:
            rec = json.load(f)
        h = hashlib.sha256(b"".join(open(os.path.join(ROOT, src), "rb").read() for src in rec["sources"])).hexdigest()
        if h != rec["source_sha256"]:
            return None
        return rec["dram_bytes_per_context_token"] * B * L
    except Exception:
        return None


def rank_workload(name: str, rank: int):
    """The workload rank `rank` runs: the same shapes, its own seed (independent sequences)."""
    wl0 = get_config(name)
    return dataclasses.replace(wl0, seed=wl0.seed + rank)


def max_over_ranks(value: float, device) -> float:
    """The maximum of `value` over all ranks (the job's time is its slowest rank's)."""
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, ctx_tokens: int, ms_per_step: float) -> float:
    """Whole-job context tokens per second: every rank encodes its batch's context each step."""
    return world * ctx_tokens / (ms_per_step * 1e-3)


def phase2_roofline(wl, n, ms, peaks):
    """Phase-2 query partials (RoPE(Q) pre-pass + attention kernel) against both bounds: the
    query rows' products over every cached key (flop) and one read of the cache, the query and
    the per-block partials written (bytes).  The roofline time is the larger of the two."""
    T, d, Hq, Hkv = wl.T, wl.d, wl.Hq, wl.Hkv
    lens = [wl.ctx_len(bi) for bi in range(wl.B)]
    flop = sum(4.0 * d * Hq * T * (Ls + (T + 1) / 2.0) for Ls in lens)
    byts = sum((Ls + T) * Hkv * d * 2 * 2 for Ls in lens) + wl.B * T * Hq * d * 2 + n * wl.B * T * Hq * (d + 1) * 4
    t_flop = flop / (peaks["bf16"] * 1e12)
    t_byte = byts / (peaks["hbm_gbs"] * 1e9)
    sec = ms * 1e-3
    return {"attn_ms": ms, "flop": flop, "bytes": byts, "tflops": flop / sec / 1e12, "gbs": byts / sec / 1e9,
            "frac_tensor": t_flop / sec, "frac_hbm": t_byte / sec, "bound": "tensor" if t_flop >= t_byte else "hbm",
            "frac": max(t_flop, t_byte) / sec, "peaks": f"{peaks['kind']} bf16 burst {peaks['bf16']} TF/s, "
                                                       f"HBM {peaks['hbm_gbs']} GB/s"}


def merge_roofline(rows, n, d, ms, peaks):
    """The query merge (star_lse_merge over n partials): HBM-bound, n (d + 1) f32 read and a bf16
    row plus its f32 LSE written per row."""
    byts = rows * (n * (d + 1) * 4 + 2 * d + 4)
    sec = ms * 1e-3
    return {"us": ms * 1e3, "bytes": byts, "gbs": byts / sec / 1e9, "frac_hbm": byts / sec / 1e9 / peaks["hbm_gbs"]}


def _ev():
    return torch.cuda.Event(enable_timing=True)


class RawEvent:
    """A cudaEvent_t created through the CUDA runtime that torch loaded.

    The library records these itself (star_set_trace_events), which torch's Event
    wrapper does not track, so creation and elapsed time go through the runtime.
    """
    _rt = None

    @classmethod
    def rt(cls):
        if cls._rt is None:
            import ctypes
            torch.cuda.init()
            cls._rt = ctypes.CDLL("libcudart.so.12")
        return cls._rt

    def __init__(self):
        import ctypes
        h = ctypes.c_void_p()
        if self.rt().cudaEventCreate(ctypes.byref(h)) != 0:
            raise RuntimeError("cudaEventCreate failed")
        self.cuda_event = h.value

    def elapsed_time(self, other) -> float:
        import ctypes
        ms = ctypes.c_float()
        rc = self.rt().cudaEventElapsedTime(ctypes.byref(ms), ctypes.c_void_p(self.cuda_event),
                                            ctypes.c_void_p(other.cuda_event))
        if rc != 0:
            raise RuntimeError(f"cudaEventElapsedTime failed ({rc})")
        return ms.value


def _pair():
    return (RawEvent(), RawEvent())


def _tpair():
    return (_ev(), _ev())


def run_star(args, rank, world, local_rank):
    import torch.distributed as dist
    peaks = load_peaks()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = rank_workload(args.config, rank)
    run = StarRun(wl, dev)
    star = run.star

    for _ in range(max(3, args.warmup)):
        run.step()
    torch.cuda.synchronize()
    if star.star_device_status() != 0:
        raise RuntimeError("device error after warm-up")

    K = args.steps
    evs = [{"p1": _pair(), "p2": _pair(), "merge": _tpair(), "dec_span": _tpair()} for _ in range(K)]
    t0, t1 = _ev(), _ev()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        t0.record()
        for k in range(K):
            run.step(evs[k])
        t1.record()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    status = star.star_device_status()
    ms_step = max_over_ranks(t0.elapsed_time(t1), dev) / K
    # The decode attention kernel alone: one more (untimed) step with events around each launch.
    ev_dec = {"dec": [_pair() for _ in range(wl.S)]}
    run.step(ev_dec)
    torch.cuda.synchronize()

    p1_ms = statistics.mean(e["p1"][0].elapsed_time(e["p1"][1]) for e in evs)
    p2_ms = statistics.mean(e["p2"][0].elapsed_time(e["p2"][1]) for e in evs)
    merge_ms = statistics.mean(e["merge"][0].elapsed_time(e["merge"][1]) for e in evs)
    dec_kernel_ms = [ev_dec["dec"][s][0].elapsed_time(ev_dec["dec"][s][1]) for s in range(wl.S)]
    dec_step_ms = statistics.mean(e["dec_span"][0].elapsed_time(e["dec_span"][1]) for e in evs) / wl.S
    flops = wl.phase1_flops()
    tflops = flops / (p1_ms * 1e-3) / 1e12
    dec_bytes = statistics.mean(wl.decode_bytes(s) for s in range(wl.S))
    dec_gbs = dec_bytes / (statistics.mean(dec_kernel_ms) * 1e-3) / 1e9

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(run, K, max(3, args.warmup), world)

    value = job_value(world, wl.context_tokens(), ms_step)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": max(3, args.warmup),
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16; 1% of context key rows x8 where the workload says peaky)",
        "config": workload_config(wl, world),
        "phase1": {"attn_ms": p1_ms, "ctx_tok_s": wl.context_tokens() / (p1_ms * 1e-3), "tflops": tflops,
                   "frac_bf16_burst": tflops / peaks["bf16"], "frac_bf16_sustained": tflops / peaks["bf16_sustained"],
                   "frac_bf16_nominal": tflops / NOMINAL["bf16_tflops"]},
        "phase2": phase2_roofline(wl, run.shape.n, p2_ms, peaks),
        "query_merge": merge_roofline(wl.B * wl.T * wl.Hq, run.shape.n, wl.d, merge_ms, peaks),
        "decode": {"us_per_step": 1e3 * dec_step_ms, "kernel_us": 1e3 * statistics.mean(dec_kernel_ms),
                   "bytes_per_step": dec_bytes, "kernel_gbs": dec_gbs, "frac_hbm": dec_gbs / peaks["hbm_gbs"],
                   "step_gbs": dec_bytes / (dec_step_ms * 1e-3) / 1e9,
                   "frac_hbm_nominal": dec_gbs / NOMINAL["hbm_gbs"],
                   "timing": "us_per_step: the S steps' span in the timed region / S (append, attention, merge "
                             "and launch gaps); kernel_us: the attention kernel alone, one extra untimed step"},
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peaks["bf16"], "unit": "TFLOP/s",
                     "frac": tflops / peaks["bf16"], "traffic": measured_traffic(wl.B, wl.L),
                     "kernel": f"star_attn_kernel<{wl.d},0> (Phase 1, with its RoPE(Q) pre-pass)",
                     "flop_per_launch": flops, "peak_source": peaks["kind"] + " bf16 burst",
                     "peak_sustained": peaks["bf16_sustained"], "frac_sustained": tflops / peaks["bf16_sustained"]},
        "gpu_launches": run.launches_per_step * K,
        "device_status": status,
    }
    if e2e:
        line["e2e"] = e2e
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(run, args.cpu_rows)
    if rank == 0:
        line["clocks"] = clk.summary()
        print(json.dumps(line), flush=True)


E2E_MIN_STEPS = 8


def run_e2e(run, K, W, world):
    """The same step through the public API with every step's inputs copied from pinned host memory
    and its results copied back, timed end to end (device events, max over ranks).

    The copies are pipelined against the compute, as a serving loop would do it: step k+1's
    host-to-device copy runs on one stream while step k computes, and step k's results go back on a
    third stream (PCIe is full duplex).  Inputs and outputs are double-buffered on the device, and
    events order every reuse: a buffer set is refilled only after the step that read it is done, and
    an output set is rewritten only after its previous copy-back is done.  The timed region starts
    before the first copy and ends after the last copy-back, so the first step's upload and the last
    step's download (the pipeline's fill and drain) are inside it too; at least E2E_MIN_STEPS steps
    are timed so that they do not stand for the steady state."""
    import torch.distributed as dist
    wl, inp = run.wl, run.inp
    names = ["q_ctx", "k_ctx", "v_ctx", "pos_ctx", "q_query", "k_query", "v_query", "pos_query",
             "q_dec", "k_dec", "v_dec", "pos_dec"] + (["anchor_pos"] if "anchor_pos" in inp else [])
    out_names = ["o_ctx", "o_q", "lse_q", "o_dec", "lse_dec"]
    in_sets = [inp, {n: torch.empty_like(inp[n]) for n in names}]
    out_sets = [{n: getattr(run, n) for n in out_names}, {n: torch.empty_like(getattr(run, n)) for n in out_names}]
    host_in = {n: inp[n].cpu().pin_memory() for n in names}
    host_out = {n: torch.empty(getattr(run, n).shape, dtype=getattr(run, n).dtype, pin_memory=True)
                for n in out_names}
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def use(k):
        run.inp = in_sets[k % 2]
        for n in out_names:
            setattr(run, n, out_sets[k % 2][n])

    def steps(n_steps):
        start, end = _ev(), _ev()
        done_in = [torch.cuda.Event() for _ in range(n_steps)]
        done_c = [torch.cuda.Event() for _ in range(n_steps)]
        done_out = [torch.cuda.Event() for _ in range(n_steps)]
        start.record(comp)
        s_in.wait_event(start)

        def load(k):
            if k >= 2:
                s_in.wait_event(done_c[k - 2])  # the step that last read this input set is done
            with torch.cuda.stream(s_in):
                for n in names:
                    in_sets[k % 2][n].copy_(host_in[n], non_blocking=True)
            done_in[k].record(s_in)

        load(0)
        for k in range(n_steps):
            if k + 1 < n_steps:
                load(k + 1)
            comp.wait_event(done_in[k])
            if k >= 2:
                comp.wait_event(done_out[k - 2])  # this output set's previous copy-back is done
            use(k)
            run.step()
            done_c[k].record(comp)
            s_out.wait_event(done_c[k])
            with torch.cuda.stream(s_out):
                for n in out_names:
                    host_out[n].copy_(out_sets[k % 2][n], non_blocking=True)
            done_out[k].record(s_out)
        comp.wait_event(done_out[n_steps - 1])
        end.record(comp)
        return start, end

    n = max(K, E2E_MIN_STEPS)
    steps(W)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t0, t1 = steps(n)
    torch.cuda.synchronize()
    use(0)
    ms = max_over_ranks(t0.elapsed_time(t1) / n, run.dev)
    return {"value": job_value(world, wl.context_tokens(), ms), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms, "steps": n,
            "copies": "pipelined: step k+1's inputs upload and step k's results download while step k computes; "
                      "the first upload and the last download are inside the timed region"}


# ---------------------------------------------------------------------------
# CPU oracle timing
# ---------------------------------------------------------------------------
def _blas_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max((i.get("num_threads", 1) for i in info), default=1)
    except Exception:
        return os.cpu_count() or 1


class OracleSample:
    """The CPU oracle, as it stands, timed on bounded pieces of one sequence's step.

    Pieces: the roped cache (the context's K through RoPE and the bf16 rounding: the KV
    append of Phase 1), Phase-1 output rows (``phase1_rows``), the first query tokens'
    per-block partials plus their merge, and one decode step over the whole cache.  The
    whole step is extrapolated from their per-unit times, for every sequence of the batch:
    cache + L_s rows + T query tokens + S decode steps; the work per unit barely changes
    over a step (decode steps add S << L keys), so the extrapolation is linear.
    """

    def __init__(self, wl, inp, bi=0):
        import numpy as np
        self.np, self.wl, self.bi = np, wl, bi
        f64 = lambda t: t.float().cpu().numpy().astype(np.float64)
        i64 = lambda t: t.cpu().numpy().astype(np.int64)
        Ls = wl.ctx_len(bi)
        self.Ls = Ls
        self.q_ctx = inp["q_ctx"][bi]                       # rows are converted when sampled
        self.k, self.v = f64(inp["k_ctx"][bi][:Ls]), f64(inp["v_ctx"][bi][:Ls])
        self.pos = i64(inp["pos_ctx"][bi][:Ls])
        self.apos = i64(inp["anchor_pos"][bi]) if "anchor_pos" in inp else None
        self.qq, self.kq, self.vq = f64(inp["q_query"][bi]), f64(inp["k_query"][bi]), f64(inp["v_query"][bi])
        self.pos_q = i64(inp["pos_query"][bi])
        self.qd, self.kd, self.vd = f64(inp["q_dec"][0, bi]), f64(inp["k_dec"][0, bi]), f64(inp["v_dec"][0, bi])
        self.pos_d = int(inp["pos_dec"][0, bi])
        self.acc = {"rows": [0.0, 0], "query": [0.0, 0], "decode": [0.0, 0]}
        self.t_cache = None
        self.ck = self.ck_full = self.cv_full = None

    def cache(self):
        import oracle
        t = time.perf_counter()
        self.ck = oracle.rope_bf16(self.k, self.pos, self.wl.theta)
        self.t_cache = time.perf_counter() - t
        self.ck_full, self.cv_full = oracle.append_tail(self.ck, self.v, self.kq, self.vq, self.pos_q, self.wl.theta)

    def rows(self, blocks, per_block, seed):
        import oracle
        np, wl = self.np, self.wl
        rng = np.random.default_rng(seed)
        rows = []
        for i in blocks:
            lo, hi = i * wl.b, min((i + 1) * wl.b, self.Ls)
            if hi > lo:
                rows.append(lo + rng.choice(hi - lo, min(per_block, hi - lo), replace=False))
        rows = np.sort(np.concatenate(rows))
        q = self.q_ctx[torch.from_numpy(rows).to(self.q_ctx.device)].float().cpu().numpy().astype(np.float64)
        t = time.perf_counter()
        oracle.phase1_rows(rows, q, self.k, self.v, self.pos, wl.b, wl.theta, wl.anchor or None, self.apos)
        self._add("rows", time.perf_counter() - t, len(rows))

    def query(self, tokens):
        """The first `tokens` query tokens: their per-block partials over the cache with the tail
        up to them, and the merge (exactly the work of those tokens)."""
        import oracle
        wl, L = self.wl, self.Ls
        ck, cv = self.ck_full[: L + tokens], self.cv_full[: L + tokens]
        t = time.perf_counter()
        Op, Lp = oracle.phase2_partials(self.qq[:tokens], self.pos_q[:tokens], ck, cv, L, wl.b, wl.theta,
                                        -(-wl.L // wl.b))
        oracle.lse_merge(Op, Lp)
        self._add("query", time.perf_counter() - t, tokens)

    def decode(self):
        import oracle
        t = time.perf_counter()
        oracle.decode_step(self.qd, self.kd, self.vd, self.pos_d, self.ck_full, self.cv_full, self.wl.theta)
        self._add("decode", time.perf_counter() - t, 1)

    def _add(self, key, sec, units):
        self.acc[key][0] += sec
        self.acc[key][1] += units

    def per_unit(self, key):
        sec, units = self.acc[key]
        return sec / units

    def step_seconds(self):
        """Extrapolated seconds of one whole step for the batch (every sequence at this one's rates)."""
        wl = self.wl
        return sum(self.t_cache * wl.ctx_len(bi) / self.Ls + wl.ctx_len(bi) * self.per_unit("rows")
                   + wl.T * self.per_unit("query") + wl.S * self.per_unit("decode") for bi in range(wl.B))

    def describe(self):
        return (f"float64 oracle on sequence {self.bi} of {self.wl.name}: roped cache {self.t_cache:.3g} s; "
                f"{self.acc['rows'][1]} Phase-1 rows (phase1_rows) at {self.per_unit('rows'):.3g} s/row; "
                f"{self.acc['query'][1]} query tokens (partials + merge) at {self.per_unit('query'):.3g} s/token; "
                f"{self.acc['decode'][1]} decode steps at {self.per_unit('decode'):.3g} s/step; value = context "
                f"tokens / the EXTRAPOLATED whole step ({self.step_seconds():.4g} s = cache + L rows + T query "
                f"tokens + S decode steps per sequence)")


def cpu_baseline(run, rows_per_block):
    wl = run.wl
    t0 = time.perf_counter()
    o = OracleSample(wl, run.inp)
    o.cache()
    o.rows(range(-(-o.Ls // wl.b)), rows_per_block, seed=0)
    o.query(min(4, wl.T))
    o.decode()
    step = o.step_seconds()
    return {"value": wl.context_tokens() / step, "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
            "sample": o.describe() + f"; sample wall time {time.perf_counter() - t0:.1f} s",
            "extrapolated_step_s": step}


def run_reference(args, rank, world):
    """The reference arm: the oracle as it stands on the host cores.  Each step is a bounded
    sample of the workload's step (2 Phase-1 rows of one block, the first query token, one
    decode step); the value is context tokens per second of the whole step extrapolated from
    the accumulated per-unit times, the unit and quantity of the CUDA arm."""
    if rank != 0:
        return
    wl = get_config(args.config)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = make_inputs(wl, dev)
    o = OracleSample(wl, inp)
    del inp
    o.cache()
    n_blocks = -(-o.Ls // wl.b)
    W = max(3, args.warmup)

    def one(k, seed):
        o.rows([k % n_blocks], 2, seed)
        o.query(1)
        o.decode()

    for w in range(W):
        one(w, w)
    o.acc = {key: [0.0, 0] for key in o.acc}
    t0 = time.perf_counter()
    for k in range(args.steps):
        one(k, 100 + k)
    sample_s = (time.perf_counter() - t0) / args.steps
    step = o.step_seconds()
    value = wl.context_tokens() / step
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": W, "ms_per_step": 1e3 * sample_s, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (same seeded inputs as the CUDA arm)",
        "config": workload_config(wl, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
                         "sample": "each step: 2 Phase-1 rows of one block, the first query token's partials and "
                                   "merge, one decode step; ms_per_step is that sample's time; " + o.describe(),
                         "extrapolated_step_s": step},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_oracle_full(args):
    """The whole oracle (Phase 1, query partials and merge, every decode step) on the full
    workload, timed on the host cores; for the small workloads whose full run takes minutes."""
    import oracle
    wl = get_config(args.config)
    inp = make_inputs(wl, "cpu")
    host = {k: (v.float().numpy().astype("float64") if v.dtype == torch.bfloat16 else v.numpy().astype("int64"))
            for k, v in inp.items()}
    t = time.perf_counter()
    oracle.run_star(host, wl.L, wl.b, wl.theta, anchor=wl.anchor or None)
    sec = time.perf_counter() - t
    print(json.dumps({"oracle_full": wl.name, "seconds": sec, "ctx_tok_s": wl.context_tokens() / sec,
                      "cores": _blas_threads(), "nproc": os.cpu_count()}), flush=True)


def run_layers(args):
    """Context encoding through `args.layers` layers on one GPU: per layer the caller's
    projections (random bf16 weights, cuBLAS through torch, in the layer callback) and the
    library's Phase 1 (RoPE + KV append + anchor-augmented attention).  One step = the
    whole stack over the workload's context; inputs resident in HBM."""
    import block_sparse_attention_star_b200 as star
    from synth import layer_inputs
    wl = get_config(args.config)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    nl, B, L, Hq, Hkv, d = args.layers, wl.B, wl.L, wl.Hq, wl.Hkv, wl.d
    hidden = Hq * d
    x0, ws = layer_inputs(wl.seed, nl, B, L, hidden, Hq * d, Hkv * d, device=dev)
    shape = workload_shape(dataclasses.replace(wl, seq_lens=None))
    caches = [star.PagedKVCache(shape, device=dev) for _ in range(nl)]
    pos = torch.arange(L, dtype=torch.int32, device=dev).repeat(B, 1).contiguous()
    x = x0.clone()
    q = torch.empty((B, L, Hq, d), dtype=torch.bfloat16, device=dev)
    k = torch.empty((B, L, Hkv, d), dtype=torch.bfloat16, device=dev)
    v, o = torch.empty_like(k), torch.empty_like(q)

    def model(layer, stage, x, q, k, v, o):
        wq, wk, wv, wo = ws[layer]
        xf = x.view(B * L, hidden)
        if stage == star.STAR_LAYER_QKV:
            torch.matmul(xf, wq, out=q.view(B * L, Hq * d))
            torch.matmul(xf, wk, out=k.view(B * L, Hkv * d))
            torch.matmul(xf, wv, out=v.view(B * L, Hkv * d))
        else:
            xf.add_(torch.matmul(o.view(B * L, Hq * d), wo))

    def step(attn_ev=None):
        x.copy_(x0)
        if attn_ev:
            star.star_set_trace_events(*attn_ev)
        star.star_encode_layers(shape, caches, pos, x, q, k, v, o, model)
        if attn_ev:
            star.star_set_trace_events(None, None)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    K = args.steps
    t0, t1 = _ev(), _ev()
    t0.record()
    for _ in range(K):
        step()
    t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / K
    attn = _pair()  # the last layer's Phase 1 (each layer re-records the pair), one extra untimed step
    step(attn)
    torch.cuda.synchronize()
    attn_ms = attn[0].elapsed_time(attn[1])
    status = star.star_device_status()
    proj_flop = 2.0 * B * L * hidden * (Hq * d + 2 * Hkv * d) + 2.0 * B * L * Hq * d * hidden
    line = {"metric": f"context encoding through {nl} layers (ctx tok/s)", "value": wl.context_tokens() / (ms * 1e-3),
            "unit": UNIT, "n_gpus": 1, "steps": K, "warmup": max(3, args.warmup), "ms_per_step": ms,
            "higher_is_better": True, "dtype": "bf16", "data": "synthetic (seeded N(0,1) hidden states, random weights)",
            "config": dict(workload_config(wl, 1), layers=nl, hidden=hidden),
            "per_layer_ms": ms / nl, "attention_ms_per_layer": attn_ms,
            "attention_tflops": wl.phase1_flops() / (attn_ms * 1e-3) / 1e12,
            "projection_flop_per_layer": proj_flop, "device_status": status}
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.oracle_full:
        run_oracle_full(args)
        return
    if args.layers > 0:
        run_layers(args)
        return
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        if args.shard:
            run_shard(args, rank, world, local_rank)
        else:
            run_star(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
