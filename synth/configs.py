"""Named synthetic workloads.

The shapes follow the attention layers of Llama-3.1-8B / 70B that the Star
Attention write-ups evaluate (8 KV heads, head_dim 128, GQA), the block-size
sweep of the 128K study (blocks of 4K..32K, a quarter of the context being the
recommended trade-off), and the million-token context study.  The value mix is
N(0, 1) bf16 throughout; the "peaky" workloads scale 1% of the context key rows
by 8 before rounding, which makes the softmax concentrate on a few keys.

Every workload is fully determined by its fields and ``seed``.
"""

from __future__ import annotations

import dataclasses
import math


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int          # independent sequences
    Hq: int         # query heads
    Hkv: int        # key/value heads (GQA groups)
    d: int          # head dim
    L: int          # context tokens
    b: int          # Star block size (context tokens per block)
    T: int          # query tokens
    S: int          # decode steps
    peaky: bool     # 1% of context key rows scaled by 8
    theta: float = 500000.0
    seed: int = 0
    page_tokens: int = 256
    anchor: int = 0                 # anchor size a (the first a tokens of block 1); 0 = b
    anchor_ids: str = "context"     # anchor position ids: "context" (tokens 0..a-1's own),
                                    # "offset" (per block, a seeded offset inside the prefix), "zero"
    seq_lens: tuple | None = None   # per-sequence context lengths (<= L, the capacity); None = all L

    @property
    def a(self) -> int:
        return self.anchor or self.b

    @property
    def n(self) -> int:
        return self.L // self.b

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def T_max(self) -> int:
        """Tail capacity: query tokens plus decode tokens."""
        return self.T + self.S

    @property
    def n_peaky(self) -> int:
        return int(math.floor(0.01 * self.L + 0.5)) if self.peaky else 0

    def with_block(self, b: int) -> "Workload":
        return dataclasses.replace(self, b=b, name=f"{self.name.split('-b')[0]}-b{b}")

    def phase1_pairs_per_head(self) -> int:
        """(query row, key) pairs Phase 1 computes for one head of one sequence.

        Block 1 is plain causal (b(b+1)/2 pairs); every later block sees the
        whole anchor (a*b) plus its own causal triangle.  Anchor rows are not
        recomputed, so they are not counted.
        """
        b, n, a = self.b, self.n, self.a
        tri = b * (b + 1) // 2
        return tri + (n - 1) * (a * b + tri)

    def phase1_pairs_of(self, length: int) -> int:
        """Pairs of one head of a sequence of ``length`` context tokens (the last block
        ragged when b does not divide it)."""
        b, a = self.b, self.a
        total = 0
        for i in range(-(-length // b)):
            n_i = min(b, length - i * b)
            total += n_i * (n_i + 1) // 2 + (a * n_i if i > 0 else 0)
        return total

    def context_tokens(self) -> int:
        """Context tokens of the whole batch."""
        return sum(self.ctx_len(bi) for bi in range(self.B))

    def phase1_flops(self) -> float:
        if self.seq_lens is None:
            return 4.0 * self.d * self.Hq * self.B * self.phase1_pairs_per_head()
        return 4.0 * self.d * self.Hq * sum(self.phase1_pairs_of(self.ctx_len(bi)) for bi in range(self.B))

    def ctx_len(self, bi: int) -> int:
        return self.seq_lens[bi] if self.seq_lens is not None else self.L

    def decode_bytes(self, step: int) -> int:
        """K and V bytes one decode step reads: every sequence's context, query tail, the
        tokens generated before and the new one."""
        return sum(self.ctx_len(bi) + self.T + step + 1 for bi in range(self.B)) * self.Hkv * self.d * 2 * 2


_BASE = {
    "tiny": Workload("tiny", B=1, Hq=4, Hkv=1, d=64, L=1024, b=256, T=16, S=8, peaky=False),
    "llama8b-32k": Workload("llama8b-32k", B=1, Hq=32, Hkv=8, d=128, L=32768, b=8192, T=64, S=32, peaky=True),
    "llama8b-128k": Workload("llama8b-128k-b32768", B=1, Hq=32, Hkv=8, d=128, L=131072, b=32768, T=64, S=64, peaky=True),
    "llama70b-128k": Workload("llama70b-128k", B=2, Hq=64, Hkv=8, d=128, L=131072, b=16384, T=128, S=64, peaky=False),
    "ctx-1m": Workload("ctx-1m", B=1, Hq=32, Hkv=8, d=128, L=1048576, b=131072, T=32, S=16, peaky=False),
}

CONFIGS: dict[str, Workload] = {
    "tiny": _BASE["tiny"],
    "llama8b-32k": _BASE["llama8b-32k"],
    "llama8b-128k-b32768": _BASE["llama8b-128k"],
    "llama8b-128k-b16384": _BASE["llama8b-128k"].with_block(16384),
    "llama8b-128k-b8192": _BASE["llama8b-128k"].with_block(8192),
    "llama8b-128k-b4096": _BASE["llama8b-128k"].with_block(4096),
    "llama70b-128k": _BASE["llama70b-128k"],
    "ctx-1m": _BASE["ctx-1m"],
    # anchor variants: a quarter-block anchor with per-block offset ids, a zero-reset anchor
    "llama8b-128k-b32768-a8192-offset": dataclasses.replace(_BASE["llama8b-128k"], name="llama8b-128k-b32768-a8192-offset",
                                                            anchor=8192, anchor_ids="offset"),
    "llama8b-128k-b32768-zero": dataclasses.replace(_BASE["llama8b-128k"], name="llama8b-128k-b32768-zero",
                                                    anchor_ids="zero"),
    # variable-length batch: a full 128K context beside a 100000-token one (ragged seventh block)
    "llama70b-128k-var": dataclasses.replace(_BASE["llama70b-128k"], name="llama70b-128k-var",
                                             seq_lens=(131072, 100000)),
}


def get_config(name: str) -> Workload:
    try:
        return CONFIGS[name]
    except KeyError as e:
        raise KeyError(f"unknown workload {name!r}; known: {sorted(CONFIGS)}") from e
