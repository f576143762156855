"""Counter-based seeded generator for the synthetic workloads.

Every value is a pure function of ``(seed, stream id, element index)``, so a
tensor can be drawn in any chunk order, on the CPU or on a GPU, and any slice
of it can be drawn again on its own.

Definition (written from the published algorithms, nothing else):

* SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014; the 64-bit finaliser constants as in Vigna's
  public-domain ``splitmix64.c``): the state advances by the golden-ratio
  increment ``0x9E3779B97F4A7C15`` and each output is the state passed
  through ``z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27;
  z *= 0x94D049BB133111EB; z ^= z >> 31`` (all mod 2**64).
* Counter form: output ``i`` of stream ``key`` is ``mix(key + (i + 1) * golden)``
  -- exactly the ``i``-th draw of a SplitMix64 seeded with ``key``.
* Element ``e`` of a tensor takes outputs ``2e`` and ``2e + 1``:
  ``u1 = ((a >> 11) + 1) / 2**53`` in (0, 1], ``u2 = (b >> 11) / 2**53`` in [0, 1),
  and the Box-Muller normal ``sqrt(-2 ln u1) * cos(2 pi u2)`` (Box and Muller,
  1958) in float64, rounded to bfloat16 (round to nearest even).

Torch int64 arithmetic wraps modulo 2**64 on both CPU and CUDA, which is the
modular arithmetic SplitMix64 needs; right shifts are made logical by masking.
"""

from __future__ import annotations

import math

import torch

from .configs import Workload

MASK64 = (1 << 64) - 1
GOLDEN = 0x9E3779B97F4A7C15
MIX1 = 0xBF58476D1CE4E5B9
MIX2 = 0x94D049BB133111EB

# One stream per drawn tensor.  Changing an id changes that tensor only.
STREAM_IDS = {
    "q_ctx": 1, "k_ctx": 2, "v_ctx": 3,
    "q_query": 4, "k_query": 5, "v_query": 6,
    "q_dec": 7, "k_dec": 8, "v_dec": 9,
    "peaky": 10,
    "anchor": 11,
    "x_layers": 12, "w_layers": 13,
}

_CHUNK = 1 << 24


def _s64(u: int) -> int:
    """Unsigned 64-bit value -> the int64 with the same bits."""
    u &= MASK64
    return u - (1 << 64) if u >= (1 << 63) else u


def splitmix64_reference(state: int, count: int) -> list[int]:
    """Pure-Python SplitMix64: the first ``count`` outputs from ``state``."""
    out = []
    for _ in range(count):
        state = (state + GOLDEN) & MASK64
        z = state
        z = ((z ^ (z >> 30)) * MIX1) & MASK64
        z = ((z ^ (z >> 27)) * MIX2) & MASK64
        out.append(z ^ (z >> 31))
    return out


def _mix_host(z: int) -> int:
    z &= MASK64
    z = ((z ^ (z >> 30)) * MIX1) & MASK64
    z = ((z ^ (z >> 27)) * MIX2) & MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, stream: int) -> int:
    """64-bit key of one stream: two SplitMix64 finalisations of (seed, stream)."""
    return _mix_host(_mix_host((seed * GOLDEN + 1) & MASK64) ^ (stream * MIX1 & MASK64))


def _lsr(z: torch.Tensor, s: int) -> torch.Tensor:
    return (z >> s) & ((1 << (64 - s)) - 1)


def _mix(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _lsr(z, 30)) * _s64(MIX1)
    z = (z ^ _lsr(z, 27)) * _s64(MIX2)
    return z ^ _lsr(z, 31)


def counter_u64(key: int, counters: torch.Tensor) -> torch.Tensor:
    """SplitMix64 output number ``counters`` (int64 tensor) of stream ``key``."""
    return _mix((counters + 1) * _s64(GOLDEN) + _s64(key))


def uniform_pair_u64(key: int, elem: torch.Tensor) -> tuple[torch.Tensor, torch.Tensor]:
    return counter_u64(key, 2 * elem), counter_u64(key, 2 * elem + 1)


def _normal_f64(key: int, elem: torch.Tensor) -> torch.Tensor:
    a, b = uniform_pair_u64(key, elem)
    u1 = (_lsr(a, 11) + 1).to(torch.float64) * (2.0 ** -53)
    u2 = _lsr(b, 11).to(torch.float64) * (2.0 ** -53)
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)


def gaussian_bf16(seed: int, stream: int, shape, device="cpu", out: torch.Tensor | None = None) -> torch.Tensor:
    """N(0, 1) bf16 tensor of ``shape``; element ``e`` (row-major) is draw ``e``."""
    numel = 1
    for s in shape:
        numel *= int(s)
    if out is None:
        out = torch.empty(tuple(shape), dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    key = stream_key(seed, stream)
    for start in range(0, numel, _CHUNK):
        end = min(numel, start + _CHUNK)
        elem = torch.arange(start, end, dtype=torch.int64, device=out.device)
        flat[start:end] = _normal_f64(key, elem).to(torch.bfloat16)
    return out


def peaky_rows(wl: Workload, device="cpu") -> torch.Tensor:
    """Context key rows scaled by 8: int64 ``[B, Hkv, n_peaky]``, sorted.

    For each (sequence, KV head) the ``round(0.01 L)`` token indices with the
    smallest hash are chosen: a uniform sample without replacement.
    """
    key = stream_key(wl.seed, STREAM_IDS["peaky"])
    t = torch.arange(wl.L, dtype=torch.int64, device=device)
    rows = []
    for bi in range(wl.B):
        per_head = []
        for h in range(wl.Hkv):
            hv = counter_u64(key, (bi * wl.Hkv + h) * wl.L + t)
            idx = torch.topk(hv, wl.n_peaky, largest=False).indices
            per_head.append(torch.sort(idx).values)
        rows.append(torch.stack(per_head) if per_head else torch.empty(0, 0, dtype=torch.int64, device=device))
    return torch.stack(rows)


def anchor_positions(wl: Workload, device="cpu") -> torch.Tensor:
    """The anchor's position ids per (sequence, block i >= 1), int32 [B, n-1, a].

    "zero": every id 0.  "offset": ids o + 0..a-1 with o drawn uniformly (seeded) from
    [0, i*b - a], i.e. the anchor placed inside the prefix that precedes block i."""
    B, n, b, a = wl.B, wl.n, wl.b, wl.a
    if wl.anchor_ids == "zero":
        return torch.zeros((B, n - 1, a), dtype=torch.int32, device=device)
    if wl.anchor_ids != "offset":
        raise ValueError(f"unknown anchor ids {wl.anchor_ids!r}")
    key = stream_key(wl.seed, STREAM_IDS["anchor"])
    idx = torch.arange(B * (n - 1), dtype=torch.int64, device=device)
    u = counter_u64(key, idx) & ((1 << 62) - 1)
    span = (idx % (n - 1) + 1) * b - a + 1          # block i = idx % (n-1) + 1
    off = (u % span).view(B, n - 1, 1)
    return (off + torch.arange(a, dtype=torch.int64, device=device)).to(torch.int32).contiguous()


def layer_inputs(seed: int, n_layers: int, B: int, L: int, hidden: int, q_width: int, kv_width: int,
                 device="cpu") -> tuple[torch.Tensor, list[tuple[torch.Tensor, ...]]]:
    """Hidden states and random per-layer weights for the multi-layer tests.

    x0: [B, L, hidden] N(0, 1) bf16.  Per layer: Wq [hidden, q_width], Wk and Wv
    [hidden, kv_width], Wo [q_width, hidden], N(0, 1) bf16 draws times a power of two
    close to 1/sqrt(fan-in) (exact in bf16), drawn in that order from one stream.
    """
    x0 = gaussian_bf16(seed, STREAM_IDS["x_layers"], (B, L, hidden), device)
    shapes = [(hidden, q_width), (hidden, kv_width), (hidden, kv_width), (q_width, hidden)]
    per = sum(a * b for a, b in shapes)
    flat = gaussian_bf16(seed, STREAM_IDS["w_layers"], (n_layers * per,), device)
    ws, off = [], 0
    for _ in range(n_layers):
        mats = []
        for fan_in, fan_out in shapes:
            scale = 2.0 ** -round(math.log2(math.sqrt(fan_in)))
            mats.append((flat[off:off + fan_in * fan_out].view(fan_in, fan_out) * scale).contiguous())
            off += fan_in * fan_out
        ws.append(tuple(mats))
    return x0, ws


def make_inputs(wl: Workload, device="cpu", parts=("ctx", "query", "dec")) -> dict[str, torch.Tensor]:
    """All inputs of one workload (bf16 values, int32 positions)."""
    B, L, T, S, Hq, Hkv, d = wl.B, wl.L, wl.T, wl.S, wl.Hq, wl.Hkv, wl.d
    g = {}
    if "ctx" in parts:
        g["q_ctx"] = gaussian_bf16(wl.seed, STREAM_IDS["q_ctx"], (B, L, Hq, d), device)
        g["k_ctx"] = gaussian_bf16(wl.seed, STREAM_IDS["k_ctx"], (B, L, Hkv, d), device)
        g["v_ctx"] = gaussian_bf16(wl.seed, STREAM_IDS["v_ctx"], (B, L, Hkv, d), device)
        if wl.peaky:
            rows = peaky_rows(wl, device)
            for bi in range(B):
                for h in range(Hkv):
                    g["k_ctx"][bi, rows[bi, h], h, :] *= 8
        g["pos_ctx"] = torch.arange(L, dtype=torch.int32, device=device).repeat(B, 1).contiguous()
        if wl.anchor_ids != "context" and wl.n > 1:
            g["anchor_pos"] = anchor_positions(wl, device)
    # Each sequence's query and generated tokens follow its own context.
    ends = torch.tensor([wl.ctx_len(bi) for bi in range(B)], dtype=torch.int32, device=device)
    if wl.seq_lens is not None:
        g["seq_len"] = ends.clone()
    if "query" in parts:
        g["q_query"] = gaussian_bf16(wl.seed, STREAM_IDS["q_query"], (B, T, Hq, d), device)
        g["k_query"] = gaussian_bf16(wl.seed, STREAM_IDS["k_query"], (B, T, Hkv, d), device)
        g["v_query"] = gaussian_bf16(wl.seed, STREAM_IDS["v_query"], (B, T, Hkv, d), device)
        g["pos_query"] = (ends[:, None] + torch.arange(T, dtype=torch.int32, device=device)[None, :]).contiguous()
    if "dec" in parts:
        g["q_dec"] = gaussian_bf16(wl.seed, STREAM_IDS["q_dec"], (S, B, 1, Hq, d), device)
        g["k_dec"] = gaussian_bf16(wl.seed, STREAM_IDS["k_dec"], (S, B, 1, Hkv, d), device)
        g["v_dec"] = gaussian_bf16(wl.seed, STREAM_IDS["v_dec"], (S, B, 1, Hkv, d), device)
        g["pos_dec"] = (T + torch.arange(S, dtype=torch.int32, device=device)[:, None] + ends[None, :]).contiguous()
    return g
