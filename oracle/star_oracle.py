"""Star Attention, restated in plain float64 numpy -- TEST INFRASTRUCTURE ONLY.

Sources (cited by page title and section throughout):

* [SA1] "Star Attention 完全拆解(一):锚点块、分块上下文编码与两阶段全局注意力"
  (pinghaoyang.com.cn) -- sections "问题定义与记号", "Phase 1: 被增广的上下文",
  "局部注意力与 KV 丢弃", "仓库里的真实实现", "Phase 2: 局部注意力与本地统计量",
  "组装全局结果", "数值稳定性:为什么实际实现用的是 log-sum-exp",
  "长上下文推理到底贵在哪里", "通信量:每层每 token 一个标量加一个向量".
* [SA2] "Star Attention: Efficient LLM Inference over Long Sequences" (abstract).
* [LCR] long-context attention review (heloowird.com), section "FlashAttention"
  (online softmax with running max m and running sum l).

What is computed (one attention layer; the caller's Q/K/V are the layer's
projections):

1. The context c = [c_1 .. c_n] of L = n*b tokens is split into blocks of b
   tokens.  Block c_i (i > 1) is prefixed by a copy of the anchor block c_1; the
   anchor keeps its own position ids and c_i keeps its own ([SA1] "Phase 1:
   被增广的上下文").  ``augmented_context`` builds c' literally.
2. RoPE (rotate-half pairing (x_j, x_{j+d/2}), inv_freq_j = theta^(-2j/d), exact
   float64 angle) is applied to Q and K of every c' token at its position id, and
   the rotated values are rounded to bf16 -- the declared rounding point, since
   the cache and the matmul operands are bf16.
3. Each augmented block runs its own causal softmax attention with scale 1/sqrt(d)
   and GQA head map kv = h // (Hq/Hkv); only the c_i rows' outputs and the c_i
   K/V are kept, the anchor's are dropped ([SA1] "局部注意力与 KV 丢弃").
4. Phase 2: query tokens take positions [L, L+T) ([SA1] "Phase 2: 局部注意力与本地
   统计量") and their K/V are appended to the tail of the last block (only the
   last host appends: [SA1] "仓库里的真实实现").  Each block gives a local
   (A_h, s_h) -- here as (O_i, LSE_i = log s_i) -- and the partials are merged by
   the softmax-statistics aggregation, which is exact global attention ([SA1]
   "组装全局结果"), computed in the log-sum-exp form of [SA1] "数值稳定性".
5. Decode: every generated token repeats step 4 against the whole cache,
   including its own K/V ([SA2] abstract: query and response tokens attend to all
   prior cached tokens).

Readings taken where the pages are silent or disagree: softmax scale 1/sqrt(d)
(the one of [SA1] "Phase 2: 局部注意力与本地统计量"); plain RoPE with theta =
500000, rotate-half pairing and no frequency scaling; the angle exact in float64;
roped Q and K rounded once to bf16; the cache holds roped K and raw V; causality by
cache index (c_i rows see the whole anchor, anchor rows only the anchor); GQA head
map kv = h // (Hq/Hkv); partials in float64 here (float32 on the GPU) with the final
O rounded to bf16; a partial with a non-finite LSE contributes nothing and a row with
none gives O = 0, LSE = -inf; the merge in max-subtracted log-sum-exp form; the
query and generated tokens' K/V at the tail of the last block, causal among
themselves, a decode token attending to itself.

Parity status per function (the pins live in ``tests/test_oracle_pins.py``):

* ``round_to_bf16``          pinned: hand-computed ties; torch's fp32->bf16 cast on fp32-exact inputs.
* ``rope_inv_freq``/``apply_rope`` pinned: complex-multiplication form, norm and
  relative-shift invariance, identity at position 0, closed-form angles.
* ``augmented_context``/``block_map`` pinned: hand-enumerated L=8, b=2 fixture; the
  anchor variants (anchor size a < b, per-block anchor position ids) by the
  hand-enumerated L=12, b=4, a=2 fixture; a ragged last block by the L=10, b=4 fixture.
* ragged / variable-length batches pinned: Phase-1 rows of a shorter context equal
  the same rows of a longer one (causality); a batch equals its sequences run
  alone; partials of missing blocks are empty and the merge equals brute force.
* ``causal_attention``       pinned: torch scaled_dot_product_attention (causal, fp64).
* ``phase1``/``phase1_rows`` pinned: n=1 equals textbook causal attention; n>1
  equals an independent full-length attention with the Star mask (library SDPA);
  with anchor variants, equals attention over each row's explicitly built key set
  (anchor keys roped at the anchor ids, own-block keys up to the row), and a
  common shift of all position ids leaves the outputs unchanged up to rounding.
* ``attend``/``phase2_partials``/``lse_merge``/``decode_step`` pinned: the merge
  equals brute-force softmax over the concatenated cache (library SDPA and
  scipy logsumexp); merge identities and overflow cases in closed form.
* ``run_star`` (the whole path) pinned in ``tests/test_oracle_path.py``: with one block it
  equals one index-causal library SDPA over the concatenated [c, q, gen]; with n > 1 its
  query and decode outputs and LSEs equal library SDPA over the independently roped,
  explicitly concatenated cache, its Phase-1 rows the full-length Star mask, its partials
  SDPA over each block's keys; per-sequence lengths likewise; decode steps that do not
  carry the cache forward, and a query tail placed before the context, are caught.
* ``encode_layers`` pinned: equals the literal per-block forward (every augmented block
  [anchor; c_i] through all layers on its own, anchor rows dropped), for a = b and a < b;
  one block equals a textbook stack of causal attention layers.
* ``kv_bytes_per_token``/``phase2_comm_bytes`` pinned: the pages' printed numbers.
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "round_to_bf16", "rope_inv_freq", "rope_angles", "apply_rope", "rope_bf16",
    "augmented_context", "block_map", "causal_attention", "attend", "phase1",
    "phase1_rows", "append_tail", "phase2_partials", "global_attention",
    "lse_merge", "decode_step", "run_star", "encode_layers", "kv_bytes_per_token",
    "phase2_comm_bytes",
]


# ----------------------------------------------------------------------------
# Rounding
# ----------------------------------------------------------------------------

def round_to_bf16(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even), as float64.

    bfloat16 keeps 8 significant bits.  With x = m * 2**e, 0.5 <= |m| < 1,
    rounding m * 2**8 to the nearest integer (numpy rounds halves to even) keeps
    exactly those bits.  Finite, normal inputs only (the workloads stay far from
    the bf16 range limits).
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.round(np.ldexp(m, 8)), e - 8)


# ----------------------------------------------------------------------------
# RoPE
# ----------------------------------------------------------------------------

def rope_inv_freq(d: int, theta: float) -> np.ndarray:
    """inv_freq_j = theta^(-2j/d), j = 0 .. d/2-1 (float64)."""
    j = np.arange(d // 2, dtype=np.float64)
    return np.power(float(theta), -2.0 * j / d)


def rope_angles(pos, d: int, theta: float) -> np.ndarray:
    """Rotation angle pos * inv_freq_j in float64, shape [N, d/2]."""
    pos = np.asarray(pos, dtype=np.float64).reshape(-1)
    return pos[:, None] * rope_inv_freq(d, theta)[None, :]


def apply_rope(x: np.ndarray, pos, theta: float) -> np.ndarray:
    """Rotate-half RoPE of x [N, H, d] at positions pos [N], float64, no rounding.

    Pair (x_j, x_{j+d/2}) turns by angle pos * inv_freq_j:
    y_j = x_j cos - x_{j+d/2} sin,  y_{j+d/2} = x_{j+d/2} cos + x_j sin.
    Scores then depend on position differences only, which is why the anchor's
    non-monotone ids are legal ([SA1] "仓库里的真实实现").
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    ang = rope_angles(pos, d, theta)[:, None, :]          # [N, 1, d/2]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., : d // 2], x[..., d // 2:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def rope_bf16(x: np.ndarray, pos, theta: float) -> np.ndarray:
    """RoPE followed by the declared bf16 rounding point."""
    return round_to_bf16(apply_rope(x, pos, theta))


# ----------------------------------------------------------------------------
# Phase 1 structure: the augmented context c' and the block map
# ----------------------------------------------------------------------------

def augmented_context(L: int, b: int, pos_ctx=None, anchor: int | None = None, anchor_pos=None) -> list[dict]:
    """c' = [c_1, (c_1 c_2), ..., (c_1 c_n)] with its position ids.

    [SA1] "Phase 1: 被增广的上下文": every block after the first is prefixed by
    the anchor c_1, which keeps ids [0, b) (here: the caller's ids of tokens
    0..b-1), while c_i keeps its own ids [(i-1)b, ib).  [SA1] "局部注意力与 KV
    丢弃": only the c_i part's KV is kept.

    Anchor variants ([SA1] "仓库里的真实实现": the anchor size is a parameter of
    its own, by default the whole first block; the implementers' notes on the
    anchor's position ids: ids sampled from the prefix range, or reset to 0):
    ``anchor`` = a <= b takes the first a tokens of c_1 as the anchor;
    ``anchor_pos`` [n-1, a] gives the anchor's position ids in block i >= 1
    (0-based), default the caller's ids of tokens 0..a-1.

    A context that is not a multiple of b ends in a ragged block: the last of
    the n = ceil(L / b) blocks holds the remaining L - (n-1) b tokens ([SA1] "问题
    定义与记号" splits the context into blocks of b tokens; the ragged tail is the
    plainest reading of a length that does not divide).

    Returns one dict per block (0-based ``i``) with ``tokens`` (context token
    index of every augmented row), ``pos`` (its position id) and ``kept`` (the
    augmented rows whose output and KV survive).
    """
    a = b if anchor is None else int(anchor)
    if not 0 < a <= b:
        raise ValueError("anchor size must be in (0, b]")
    n = -(-L // b)
    pos_ctx = np.arange(L, dtype=np.int64) if pos_ctx is None else np.asarray(pos_ctx, dtype=np.int64)
    if anchor_pos is not None:
        anchor_pos = np.asarray(anchor_pos, dtype=np.int64).reshape(n - 1, a)
    out = []
    for i in range(n):
        own = np.arange(i * b, min((i + 1) * b, L), dtype=np.int64)
        if i == 0:
            tokens, pos = own, pos_ctx[own]
        else:
            tokens = np.concatenate([np.arange(a, dtype=np.int64), own])
            apos = pos_ctx[:a] if anchor_pos is None else anchor_pos[i - 1]
            pos = np.concatenate([apos, pos_ctx[own]])
        out.append({"i": i, "tokens": tokens, "pos": pos, "kept": np.arange(len(tokens) - len(own), len(tokens))})
    return out


def block_map(L: int, b: int, page_tokens: int, page_table) -> np.ndarray:
    """token t -> (block t // b, physical page page_table[t // P], slot t % P), int64 [L, 3]."""
    t = np.arange(L, dtype=np.int64)
    page_table = np.asarray(page_table, dtype=np.int64)
    return np.stack([t // b, page_table[t // page_tokens], t % page_tokens], axis=1)


# ----------------------------------------------------------------------------
# Attention primitives
# ----------------------------------------------------------------------------

def attend(q: np.ndarray, k: np.ndarray, v: np.ndarray, visible: np.ndarray | None = None):
    """Softmax attention of rows q [M, Hq, d] over keys k, v [N, Hkv, d].

    visible: bool [M, N] (None = all keys).  Per query head h the key head is
    h // (Hq/Hkv).  Returns O [M, Hq, d] and LSE [M, Hq] = log sum_k exp(q.k/sqrt(d))
    -- the local (A_h, s_h) pair of [SA1] "Phase 2: 局部注意力与本地统计量" with
    s_h kept as its logarithm.  A row with no visible key gets O = 0, LSE = -inf.
    """
    M, Hq, d = q.shape
    N, Hkv, _ = k.shape
    G = Hq // Hkv
    scale = 1.0 / math.sqrt(d)
    O = np.zeros((M, Hq, d))
    LSE = np.full((M, Hq), -np.inf)
    if N == 0:
        return O, LSE
    for h in range(Hq):
        kv = h // G
        s = (q[:, h, :] @ k[:, kv, :].T) * scale            # [M, N]
        if visible is not None:
            s = np.where(visible, s, -np.inf)
        m = np.max(s, axis=1, keepdims=True)
        ok = np.isfinite(m[:, 0])
        m_safe = np.where(np.isfinite(m), m, 0.0)
        p = np.exp(s - m_safe)
        l = p.sum(axis=1, keepdims=True)
        O[ok, h, :] = (p[ok] @ v[:, kv, :]) / l[ok]
        LSE[ok, h] = m[ok, 0] + np.log(l[ok, 0])
    return O, LSE


def causal_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray):
    """Index-causal attention over one sequence: row r sees keys 0..r."""
    N = q.shape[0]
    vis = np.tril(np.ones((N, N), dtype=bool))
    return attend(q, k, v, vis)


# ----------------------------------------------------------------------------
# Phase 1
# ----------------------------------------------------------------------------

def phase1(q: np.ndarray, k: np.ndarray, v: np.ndarray, pos_ctx, b: int, theta: float,
           anchor: int | None = None, anchor_pos=None):
    """Phase 1 of one sequence by literally building c'.

    q [L, Hq, d], k/v [L, Hkv, d] (pre-RoPE, bf16 values held in float64).
    Returns O_ctx [L, Hq, d] (float64), and the cache: roped bf16 K [L, Hkv, d]
    and V [L, Hkv, d] -- only the c_i parts, the anchor copies are dropped.
    ``anchor``/``anchor_pos``: the anchor variants of ``augmented_context``.
    """
    L = q.shape[0]
    O = np.zeros_like(q, dtype=np.float64)
    ck = np.zeros_like(k, dtype=np.float64)
    cv = np.zeros_like(v, dtype=np.float64)
    for blk in augmented_context(L, b, pos_ctx, anchor, anchor_pos):
        tok, pos, kept = blk["tokens"], blk["pos"], blk["kept"]
        qr = rope_bf16(q[tok], pos, theta)
        kr = rope_bf16(k[tok], pos, theta)
        vv = np.asarray(v[tok], dtype=np.float64)
        Ob, _ = causal_attention(qr, kr, vv)
        own = tok[kept]
        O[own] = Ob[kept]
        ck[own] = kr[kept]
        cv[own] = vv[kept]
    return O, ck, cv


def phase1_rows(rows, q_rows: np.ndarray, k: np.ndarray, v: np.ndarray, pos_ctx, b: int, theta: float,
                anchor: int | None = None, anchor_pos=None):
    """Phase-1 outputs of selected context rows only (same definition as ``phase1``).

    rows: context token indices; q_rows [len(rows), Hq, d] their pre-RoPE queries;
    k/v [L, Hkv, d] the context keys/values.  Row t of block i = t // b is the
    augmented row of c'_i that holds token t; it sees the augmented rows before it:
    the whole anchor (its first a tokens, roped at the anchor's ids) and its own
    block up to t.
    """
    rows = np.asarray(rows, dtype=np.int64)
    L = k.shape[0]
    n = -(-L // b)
    a = b if anchor is None else int(anchor)
    pos_ctx = np.arange(L, dtype=np.int64) if pos_ctx is None else np.asarray(pos_ctx, dtype=np.int64)
    if anchor_pos is not None:
        anchor_pos = np.asarray(anchor_pos, dtype=np.int64).reshape(n - 1, a)
    out = np.zeros((len(rows),) + q_rows.shape[1:])
    cache: dict[int, np.ndarray] = {}

    def roped_block(i):
        if i not in cache:
            tok = np.arange(i * b, min((i + 1) * b, L))
            cache[i] = rope_bf16(k[tok], pos_ctx[tok], theta)
        return cache[i]

    for i in np.unique(rows // b):
        sel = np.nonzero(rows // b == i)[0]
        own = np.arange(i * b, min((i + 1) * b, L))
        keys, vals, key_idx = roped_block(i), np.asarray(v[own], dtype=np.float64), own
        if i > 0:
            apos = pos_ctx[:a] if anchor_pos is None else anchor_pos[i - 1]
            keys = np.concatenate([rope_bf16(k[:a], apos, theta), keys])
            vals = np.concatenate([np.asarray(v[:a], dtype=np.float64), vals])
            key_idx = np.concatenate([np.arange(a), own])
        # augmented row of token t sees the anchor (all of it) and its own block up to t
        vis = key_idx[None, :] <= rows[sel][:, None]
        qr = rope_bf16(q_rows[sel], pos_ctx[rows[sel]], theta)
        O, _ = attend(qr, keys, vals, vis)
        out[sel] = O
    return out


# ----------------------------------------------------------------------------
# Phase 2
# ----------------------------------------------------------------------------

def append_tail(ck: np.ndarray, cv: np.ndarray, k_new: np.ndarray, v_new: np.ndarray, pos_new, theta: float):
    """Append roped (bf16) K and V of new tokens after the cache (tail of the last block)."""
    return (np.concatenate([ck, rope_bf16(k_new, pos_new, theta)]),
            np.concatenate([cv, np.asarray(v_new, dtype=np.float64)]))


def phase2_partials(q_query: np.ndarray, pos_query, ck: np.ndarray, cv: np.ndarray, L: int, b: int, theta: float,
                    n_parts: int | None = None):
    """Per-block local attention of the query rows ([SA1] "Phase 2: 局部注意力与本地统计量").

    ck/cv: the cache [L + T, Hkv, d] with the query tokens' K/V already appended
    (tail of the last block).  Query token t (cache index L + t) sees every key of
    blocks 1..n-1 and, in the last block, its context keys plus tail keys L..L+t.
    n = ceil(L / b); with ``n_parts`` > n (a batch whose longest sequence has more
    blocks) the partials of the missing blocks are empty: O = 0, LSE = -inf, which
    the merge skips ([SA1] "数值稳定性").
    Returns O_part [n_parts, T, Hq, d] and LSE_part [n_parts, T, Hq].
    """
    T = q_query.shape[0]
    n = -(-L // b)
    n_parts = n if n_parts is None else int(n_parts)
    qr = rope_bf16(q_query, pos_query, theta)
    O_part = np.zeros((n_parts, T) + q_query.shape[1:])
    LSE_part = np.full((n_parts, T, q_query.shape[1]), -np.inf)
    row_idx = L + np.arange(T)
    for i in range(n):
        lo, hi = i * b, (i + 1) * b if i < n - 1 else ck.shape[0]
        key_idx = np.arange(lo, hi)
        vis = key_idx[None, :] <= row_idx[:, None]
        O_part[i], LSE_part[i] = attend(qr, ck[lo:hi], cv[lo:hi], vis)
    return O_part, LSE_part


def global_attention(q_roped: np.ndarray, row_idx, ck: np.ndarray, cv: np.ndarray):
    """Brute-force softmax of roped rows over the whole cache, causal by cache index."""
    key_idx = np.arange(ck.shape[0])
    vis = key_idx[None, :] <= np.asarray(row_idx)[:, None]
    return attend(q_roped, ck, cv, vis)


def lse_merge(O_parts: np.ndarray, LSE_parts: np.ndarray):
    """Merge per-block partials into global attention ([SA1] "组装全局结果", "数值稳定性").

    O_parts [n, ..., d], LSE_parts [n, ...].  The partials are folded in order with
    the pairwise update lse <- logaddexp(lse, lse_b),
    out <- e^{lse_old - lse} out + e^{lse_b - lse} out_b, which is the page's update
    rewritten so it cannot overflow.  A partial whose LSE is not finite (an empty
    block: -inf, or a NaN) is skipped; a row with no finite partial gives O = 0,
    LSE = -inf.
    """
    O_parts = np.asarray(O_parts, dtype=np.float64)
    LSE_parts = np.asarray(LSE_parts, dtype=np.float64)
    out = np.zeros(O_parts.shape[1:])
    lse = np.full(LSE_parts.shape[1:], -np.inf)
    for i in range(O_parts.shape[0]):
        lb, ob = LSE_parts[i], O_parts[i]
        use = np.isfinite(lb)
        first = use & ~np.isfinite(lse)        # first usable partial of the row: take it
        both = use & np.isfinite(lse)          # otherwise: the pairwise update
        new_lse = lse.copy()
        new_out = out.copy()
        new_lse[first] = lb[first]
        new_out[first] = ob[first]
        new_lse[both] = np.logaddexp(lse[both], lb[both])
        new_out[both] = (np.exp(lse[both] - new_lse[both])[:, None] * out[both]
                         + np.exp(lb[both] - new_lse[both])[:, None] * ob[both])
        out, lse = new_out, new_lse
    return out, lse


def decode_step(q_tok: np.ndarray, k_tok: np.ndarray, v_tok: np.ndarray, pos, ck, cv, theta: float):
    """One generated token: append its K/V, then attend over the whole cache incl. itself.

    q_tok [1, Hq, d], k_tok/v_tok [1, Hkv, d].  Returns (O [1, Hq, d], LSE [1, Hq], ck, cv).
    """
    ck, cv = append_tail(ck, cv, k_tok, v_tok, [pos], theta)
    qr = rope_bf16(q_tok, [pos], theta)
    O, LSE = global_attention(qr, [ck.shape[0] - 1], ck, cv)
    return O, LSE, ck, cv


# ----------------------------------------------------------------------------
# The whole path for one workload
# ----------------------------------------------------------------------------

def run_star(inp: dict, L: int, b: int, theta: float, with_phase1: bool = True, anchor: int | None = None) -> dict:
    """Phase 1, Phase 2 (partials + merge) and decode for every sequence.

    ``inp`` holds float64 (bf16-valued) arrays laid out like the synthetic inputs:
    q_ctx [B, L, Hq, d], k_ctx/v_ctx [B, L, Hkv, d], pos_ctx [B, L], q_query
    [B, T, Hq, d], k_query/v_query [B, T, Hkv, d], pos_query [B, T], q_dec
    [S, B, 1, Hq, d], k_dec/v_dec [S, B, 1, Hkv, d], pos_dec [S, B]; optionally
    anchor_pos [B, n-1, a] (the anchor's position ids per block, see
    ``augmented_context``) and seq_len [B] (each sequence's context length; the
    context arrays are then padded to L and the rows past a sequence's length are
    ignored, its outputs there are 0).  ``anchor``: the anchor size a (default b).
    Every sequence has ceil(L / b) partials; those past its own blocks are empty.
    """
    B = inp["q_ctx"].shape[0]
    res: dict[str, list] = {k: [] for k in ("o_ctx", "cache_k", "cache_v", "o_part", "lse_part",
                                            "o_query", "lse_query", "o_dec", "lse_dec")}
    n_parts = -(-L // b)
    for bi in range(B):
        Ls = int(inp["seq_len"][bi]) if inp.get("seq_len") is not None else L
        if with_phase1:
            apos = inp["anchor_pos"][bi] if inp.get("anchor_pos") is not None else None
            O1, ck, cv = phase1(inp["q_ctx"][bi][:Ls], inp["k_ctx"][bi][:Ls], inp["v_ctx"][bi][:Ls],
                                inp["pos_ctx"][bi][:Ls], b, theta, anchor, apos)
            Opad = np.zeros(inp["q_ctx"][bi].shape)
            Opad[:Ls] = O1
            res["o_ctx"].append(Opad)
        else:
            tok = np.arange(Ls)
            ck = rope_bf16(inp["k_ctx"][bi][:Ls], inp["pos_ctx"][bi][tok], theta)
            cv = np.asarray(inp["v_ctx"][bi][:Ls], dtype=np.float64)
        res["cache_k"].append(ck)
        res["cache_v"].append(cv)
        ck, cv = append_tail(ck, cv, inp["k_query"][bi], inp["v_query"][bi], inp["pos_query"][bi], theta)
        Op, Lp = phase2_partials(inp["q_query"][bi], inp["pos_query"][bi], ck, cv, Ls, b, theta, n_parts)
        Oq, Lq = lse_merge(Op, Lp)
        res["o_part"].append(Op)
        res["lse_part"].append(Lp)
        res["o_query"].append(Oq)
        res["lse_query"].append(Lq)
        od, ld = [], []
        for s in range(inp["q_dec"].shape[0]):
            O, LSE, ck, cv = decode_step(inp["q_dec"][s, bi], inp["k_dec"][s, bi], inp["v_dec"][s, bi],
                                         int(inp["pos_dec"][s, bi]), ck, cv, theta)
            od.append(O[0])
            ld.append(LSE[0])
        res["o_dec"].append(np.stack(od) if od else np.zeros((0,) + inp["q_dec"].shape[3:]))
        res["lse_dec"].append(np.stack(ld) if ld else np.zeros((0, inp["q_dec"].shape[3])))
    out = {}
    for k, vals in res.items():
        if not vals:
            continue
        if k in ("o_part", "lse_part"):
            out[k] = np.stack(vals, axis=1)          # [n, B, ...]
        elif k in ("o_dec", "lse_dec"):
            out[k] = np.stack(vals, axis=1)          # [S, B, ...]
        elif k in ("cache_k", "cache_v") and len({v.shape for v in vals}) > 1:
            out[k] = vals                            # per-sequence lengths differ
        else:
            out[k] = np.stack(vals)
    return out


# ----------------------------------------------------------------------------
# Several layers ([SA1] "仓库里的真实实现")
# ----------------------------------------------------------------------------

def encode_layers(x: np.ndarray, pos_ctx, b: int, theta: float, layers, anchor: int | None = None):
    """Phase 1 of a stack of layers for one sequence, one pass over the L real tokens per layer.

    [SA1] "仓库里的真实实现": every augmented block [a_1; c_i] runs the whole model forward
    on its own (past_key_values=None), and the anchor's part of every layer's KV is
    dropped.  The anchor is the first a tokens of c_1 with c_1's position ids and the
    attention is causal, so its hidden states at every layer are c_1's first a rows;
    the layer-by-layer pass below therefore takes the anchor's keys and values of each
    layer from that layer's c_1 (through ``phase1``).  The pins check this against the
    literal per-block forward.

    x: hidden states [L, ...] (float64; the caller's layout).  layers: a list of
    (qkv_fn, out_fn) per layer, the caller's model in float64: qkv_fn(x) -> q [L, Hq, d],
    k, v [L, Hkv, d] (pre-RoPE, rounded as the caller rounds them); out_fn(x, o) -> the
    next x, from the attention output o rounded to bf16 (the output type of Phase 1).
    Returns the final x and, per layer, (o, cache K, cache V).
    """
    per_layer = []
    for qkv_fn, out_fn in layers:
        q, k, v = qkv_fn(x)
        o, ck, cv = phase1(q, k, v, pos_ctx, b, theta, anchor)
        o = round_to_bf16(o)
        per_layer.append((o, ck, cv))
        x = out_fn(x, o)
    return x, per_layer


# ----------------------------------------------------------------------------
# Byte accounting ([SA1] "长上下文推理到底贵在哪里", "通信量")
# ----------------------------------------------------------------------------

def kv_bytes_per_token(layers: int, kv_heads: int, head_dim: int, elem_bytes: int = 2) -> int:
    """K and V bytes one token adds to the cache: 2 * layers * kv_heads * head_dim * bytes."""
    return 2 * layers * kv_heads * head_dim * elem_bytes


def phase2_comm_bytes(hosts: int, layers: int, tokens: int, heads: int, head_dim: int, elem_bytes: int = 2) -> int:
    """Phase-2 (output, statistic) traffic: hosts * layers * tokens * heads * (head_dim + 1) * bytes."""
    return hosts * layers * tokens * heads * (head_dim + 1) * elem_bytes
