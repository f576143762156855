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
over ranks.  `--impl reference` times the CPU oracle (float64 numpy) on a
bounded sample of the same workload on the host cores.
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
        s.star_lse_merge(self.shape.n, wl.B * wl.T * wl.Hq, wl.d, self.o_part, self.lse_part, self.o_q, self.lse_q)
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
    evs = [{"p1": _pair(), "p2": _pair(), "dec_span": _tpair()} for _ in range(K)]
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
                   "frac_bf16_burst": tflops / peaks["bf16"], "frac_bf16_sustained": tflops / peaks["bf16_sustained"]},
        "phase2": {"attn_ms": p2_ms},
        "decode": {"us_per_step": 1e3 * dec_step_ms, "kernel_us": 1e3 * statistics.mean(dec_kernel_ms),
                   "bytes_per_step": dec_bytes, "kernel_gbs": dec_gbs, "frac_hbm": dec_gbs / peaks["hbm_gbs"],
                   "step_gbs": dec_bytes / (dec_step_ms * 1e-3) / 1e9,
                   "timing": "us_per_step: the S steps' span in the timed region / S (append, attention, merge "
                             "and launch gaps); kernel_us: the attention kernel alone, one extra untimed step"},
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peaks["bf16_sustained"], "unit": "TFLOP/s",
                     "frac": tflops / peaks["bf16_sustained"], "traffic": measured_traffic(wl.B, wl.L),
                     "kernel": f"star_attn_kernel<{wl.d},0> (Phase 1)", "flop_per_launch": flops,
                     "peak_source": peaks["kind"] + " bf16 sustained"},
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


def oracle_phase1_sample(wl, host, blocks, rows_per_block, seed=0):
    """Time the oracle's Phase-1 rows on a sample: `rows_per_block` rows of each listed block."""
    import numpy as np
    import oracle
    rng = np.random.default_rng(seed)
    rows = np.concatenate([i * wl.b + rng.choice(wl.b, rows_per_block, replace=False) for i in blocks])
    rows.sort()
    k = host["k"].float().numpy().astype(np.float64)
    v = host["v"].float().numpy().astype(np.float64)
    q = host["q"][rows].float().numpy().astype(np.float64)
    pos = host["pos"].numpy().astype(np.int64)
    apos = host["anchor_pos"].numpy().astype(np.int64) if host.get("anchor_pos") is not None else None
    t = time.perf_counter()
    oracle.phase1_rows(rows, q, k, v, pos, wl.b, wl.theta, wl.anchor or None, apos)
    return len(rows), time.perf_counter() - t


def _host_seq0(inp):
    return {"q": inp["q_ctx"][0].cpu(), "k": inp["k_ctx"][0].cpu(), "v": inp["v_ctx"][0].cpu(),
            "pos": inp["pos_ctx"][0].cpu(),
            "anchor_pos": inp["anchor_pos"][0].cpu() if "anchor_pos" in inp else None}


def cpu_baseline(run, rows_per_block):
    wl = run.wl
    host = _host_seq0(run.inp)
    nrows, sec = oracle_phase1_sample(wl, host, range(wl.n), rows_per_block)
    return {"value": nrows / sec, "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
            "sample": f"float64 oracle, Phase-1 output of {nrows} context rows ({rows_per_block} per block, all "
                      f"{wl.Hq} heads, sequence 0) of {wl.name}; value = rows/s; {sec:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    wl = get_config(args.config)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = make_inputs(wl, dev, parts=("ctx",))
    host = _host_seq0(inp)
    del inp
    rows_per_block = 4
    W = max(3, args.warmup)
    for w in range(W):
        oracle_phase1_sample(wl, host, [w % wl.n], rows_per_block, seed=w)
    tot_rows, tot_sec = 0, 0.0
    for k in range(args.steps):
        r, s = oracle_phase1_sample(wl, host, [k % wl.n], rows_per_block, seed=100 + k)
        tot_rows += r
        tot_sec += s
    value = tot_rows / tot_sec
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": W, "ms_per_step": 1e3 * tot_sec / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (same seeded inputs as the CUDA arm)",
        "config": workload_config(wl, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
                         "sample": f"each step: float64 oracle Phase-1 output of {rows_per_block} context rows of one "
                                   f"block (all {wl.Hq} heads) of {wl.name}; value = rows/s"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


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
    if args.layers > 0:
        run_layers(args)
        return
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        run_star(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
