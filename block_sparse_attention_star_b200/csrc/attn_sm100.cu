// Star Attention tensor-core attention for sm_100a (tcgen05 + TMEM + TMA).
//
// One kernel serves two steps of the hot path:
//
//  * mode 0 -- Phase 1, anchor-augmented blockwise-local causal attention
//    ("Star Attention 完全拆解(一)", Phase 1: "被增广的上下文" and "局部注意力与
//    KV 丢弃").  Query row t of block i > 1 attends to the anchor keys [0, b)
//    and to its own block's keys up to itself; block 1 is plain causal.  The
//    anchor is never materialised: its keys are block 1's cached pages (the
//    anchor keeps block 1's positions, so its roped K/V equal block 1's bit for
//    bit), and anchor rows are never recomputed (their outputs are discarded).
//  * mode 1 -- Phase 2, the query tokens' local attention against each block
//    ("Phase 2: 局部注意力与本地统计量"), written as per-part (O, LSE) partials
//    for the exact log-sum-exp merge ("组装全局结果", "数值稳定性").  A part is a
//    chunk of one block; the last block's last chunk also covers the query tail.
//
// Both are "causal by cache index over a key set": a work item lists up to two
// runs of 128-key tiles, and a key is visible to a row iff its cache index is
// <= the row's cache index.
//
// CTA organisation (384 threads, persistent, one CTA per SM):
//   warp 0      TMA producer: K and V tiles from the paged cache into two
//               shared-memory rings (128-byte swizzle; each CTA loads its own tiles).
//   warp 1      MMA issuer: S_w = Q_w K^T (SS form) and O_w += P_w V (A from TMEM).
//   warps 4-7   softmax warpgroup 0 (Q tile 0: rows <-> TMEM lanes 0..127)
//   warps 8-11  softmax warpgroup 1 (Q tile 1)
// The two Q tiles of an item share every K/V tile (two heads of one GQA group in
// Phase 1; two row tiles of the group in Phase 2), so each K/V byte staged in
// shared memory feeds 2 x 128 query rows.  While warpgroup 0 turns S_0 into
// P_0 the tensor core runs warpgroup 1's products, and vice versa.
//
// TMEM (512 columns): S_0 [0,128), S_1 [128,256), O_0 [256,256+d), O_1 [384,384+d).
// P_w (bf16, two per 32-bit column) overwrites the first 64 columns of S_w.
// Softmax uses the online (running max m, running sum l) formulation of the
// FlashAttention section of the long-context attention review, in base 2 with a
// lazily updated max: O and l are rescaled only when the tile max exceeds the
// running max by more than 32 (so P <= 2^32: bf16 and f32 hold it with the same
// relative precision as P <= 1, and a row's f32 sums stay below 2^52 for up to
// 2^20 keys, far from overflow).
#include "common.cuh"
#include "internal.h"

#include <algorithm>
#include <climits>
#include <cstring>

namespace star {

namespace {

constexpr int kThreads = 384;
constexpr int kRows = 128;        // rows per Q tile (UMMA M)
constexpr int kKeys = 128;        // keys per K/V tile (UMMA N of QK^T, K of PV)
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 32.0f;
// Per-warpgroup register budgets (setmaxnreg), chosen so neither role spills;
// 128 x ctl + 256 x softmax must stay within the 384 x 168 registers of the launch.
template <int D>
struct RegSplit {
  static constexpr uint32_t kCtl = (D == 128) ? 104 : 72;
  static constexpr uint32_t kSoftmax = (D == 128) ? 200 : 216;
  static_assert(128 * kCtl + 256 * kSoftmax <= kThreads * 168, "register split exceeds the launch budget");
};

struct Params {
  const bf16* q;  // rotated queries (RoPE applied by the pre-pass)
  bf16* out_bf16;
  float* out_f32;
  float* lse_f32;
  const int32_t* page_table;
  int max_pages, num_pages, P;
  int B, Hq, Hkv, G, L, b, n, Ntok;
  // Phase-2 tiling
  int chunk_keys, chunks_per_block, tail_tiles, TQ, HT, NTT, NHT, npairs;
  int num_items;
  // Phase-1 anchor: its size, and whether its keys come from the tmKA map (roped at caller ids)
  int anchor, anchor_k_on;
  // Block range [blk0, blk0 + nblk) of every sequence (a shard; the whole context by
  // default); tail_on: the range holds the query tail.  Mode 0 reads q and writes out as
  // rows [0, Lrows) per sequence, row r holding context token r + row_off.
  int blk0, nblk, tail_on, row_off, Lrows;
  SeqShift sh;  // per-sequence context lengths L + delta[bi] (sh.on = 0: every sequence has L)
  float scale_log2;
};

struct Item {
  int bi, g;
  int a_start, a_tiles;   // first run of key tiles (cache index of its first key, tile count)
  int a_end;              // keys of the first run at or past a_end are not visible
  int b_start, b_tiles;   // second run (tiles start at b_start rounded down to 128)
  int skip;               // mode 0: the item's rows are all past the sequence's context
  int part;               // Phase 2: output part (global chunk index)
  int r0;                 // Phase 1: context index of the tile's first row
  int hp;                 // Phase 1: head pair in the group; Phase 2: row-tile pair
};

// Work items.  Phase 1, per (sequence, KV head): items of blocks 2..n first,
// then block 1's, each run ordered by descending q-tile, so item cost falls
// monotonically and the round-robin assignment to CTAs stays balanced.
__device__ __forceinline__ int ctx_len(const Params& p, int bi) { return p.L + (p.sh.on ? p.sh.delta[bi] : 0); }

template <int MODE>
__device__ __forceinline__ Item decode_item(const Params& p, int idx) {
  Item it;
  it.skip = 0;
  if (MODE == 0) {
    const int nqt = p.b / kRows;
    const int npairs = p.G / 2;
    const int per_group = p.nblk * nqt * npairs;
    const int grp = idx / per_group;
    int w = idx - grp * per_group;
    it.bi = grp / p.Hkv;
    it.g = grp - it.bi * p.Hkv;
    const int has_first = p.blk0 == 0;         // the range holds the context's first block
    const int n_later = p.nblk - has_first;    // blocks with the anchor in front
    const int nonanchor = n_later * nqt * npairs;
    int t, i;
    if (w < nonanchor) {
      const int per_t = n_later * npairs;
      t = nqt - 1 - w / per_t;
      const int rem = w - (w / per_t) * per_t;
      i = p.blk0 + has_first + rem / npairs;
      it.hp = rem - (rem / npairs) * npairs;
    } else {
      w -= nonanchor;
      t = nqt - 1 - w / npairs;
      i = 0;
      it.hp = w - (w / npairs) * npairs;
    }
    it.a_start = 0;
    it.a_tiles = (i > 0) ? p.anchor / kRows : 0;  // the anchor: the first a keys of block 1
    it.a_end = p.anchor;
    it.b_start = i * p.b;
    it.b_tiles = t + 1;
    it.part = i;
    it.r0 = i * p.b + t * kRows;
    it.skip = it.r0 >= ctx_len(p, it.bi);  // a shorter sequence: every row of the tile is padding
  } else {
    it.hp = idx % p.npairs;
    int rest = idx / p.npairs;
    it.g = rest % p.Hkv;
    rest /= p.Hkv;
    it.bi = rest % p.B;
    const int c = p.blk0 * p.chunks_per_block + rest / p.B;  // the chunk's index in the context
    const int Ls = ctx_len(p, it.bi);
    it.part = c - p.blk0 * p.chunks_per_block;
    // The chunk's context keys, cut at the sequence's length; the tail (query tokens,
    // cache indices Ls ..) follows the chunk that holds the last context key.
    it.a_start = c * p.chunk_keys;
    it.a_end = min(it.a_start + p.chunk_keys, Ls);
    it.a_tiles = it.a_end > it.a_start ? (it.a_end - it.a_start + kKeys - 1) / kKeys : 0;
    const bool last = p.tail_on && (c == (Ls - 1) / p.chunk_keys);
    it.b_start = Ls;
    it.b_tiles = last ? (Ls % kKeys + p.Ntok + kKeys - 1) / kKeys : 0;
    it.r0 = 0;
  }
  return it;
}

__device__ __forceinline__ int tile_key0(const Item& it, int j) {
  return j < it.a_tiles ? it.a_start + j * kKeys : (it.b_start & ~(kKeys - 1)) + (j - it.a_tiles) * kKeys;
}

struct RowInfo {
  bool valid;
  int head;       // query head
  int tok;        // index into q / outputs
  int cache_idx;  // cache index used by the causal rule
};

template <int MODE>
__device__ __forceinline__ RowInfo row_info(const Params& p, const Item& it, int wg, int row) {
  RowInfo r;
  if (MODE == 0) {
    r.valid = true;
    r.head = it.g * p.G + 2 * it.hp + wg;
    r.tok = it.r0 + row;
    r.cache_idx = r.tok;
  } else {
    const int rt = 2 * it.hp + wg;
    const int ht = rt / p.NTT, tt = rt - (rt / p.NTT) * p.NTT;
    const int hl = ht * p.HT + row / p.TQ;
    const int t = tt * p.TQ + (row % p.TQ);
    r.valid = (rt < p.NTT * p.NHT) && (hl < p.G) && (t < p.Ntok);
    r.head = it.g * p.G + (r.valid ? hl : 0);
    r.tok = r.valid ? t : 0;
    r.cache_idx = r.valid ? ctx_len(p, it.bi) + t : INT_MAX;
  }
  if (!r.valid) r.cache_idx = INT_MAX;
  return r;
}

// One thread copies its Q row (already rotated, bf16) into the K-major
// 128-byte-swizzled tile: element (row, col) lives in the 64-column atom col/64
// at byte row*128 + 16*((col%64/8) ^ (row%8)) + 2*(col%8).  Rows past the
// queries are zeros.
template <int D>
__device__ __forceinline__ void load_q_row(const Params& p, const Item& it, const RowInfo& r, uint8_t* sQ, int row) {
  const bf16* src = p.q + (((size_t)it.bi * p.Ntok + r.tok) * p.Hq + r.head) * D;
  uint4 v[D / 8];
#pragma unroll
  for (int c = 0; c < D / 8; ++c) v[c] = r.valid ? __ldg(reinterpret_cast<const uint4*>(src) + c) : make_uint4(0, 0, 0, 0);
#pragma unroll
  for (int c = 0; c < D / 8; ++c) {
    const int atom = c / 8, chunk = c % 8;
    *reinterpret_cast<uint4*>(sQ + atom * (kRows * 128) + row * 128 + ((chunk ^ (row & 7)) * 16)) = v[c];
  }
}

template <int D, int MODE, int NSK, int NSV>
struct Smem {
  static constexpr int kTile = kRows * D * 2;  // bytes of one 128 x D bf16 tile
  static constexpr int kQ0 = 0;
  static constexpr int kK = 2 * kTile;
  static constexpr int kV = kK + NSK * kTile;
  static constexpr int kBar = kV + NSV * kTile;
  static constexpr int kNumBars = 2 * NSK + 2 * NSV + 2 + 2 + 4 + 2 + 1 + 2 + 1;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kEnd = kTmemSlot + 16;
  static constexpr int kBytes = kEnd + 1024;  // slack for 1024-byte alignment
};

template <int D, int MODE, int NSK, int NSV>
__global__ void __launch_bounds__(kThreads, 1)
    star_attn_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKA,
                     const __grid_constant__ Params p) {
  using S = Smem<D, MODE, NSK, NSV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
  uint64_t* k_full = bars;
  uint64_t* k_empty = k_full + NSK;
  uint64_t* v_full = k_empty + NSK;
  uint64_t* v_empty = v_full + NSV;
  uint64_t* q_full = v_empty + NSV;   // [2]
  uint64_t* s_full = q_full + 2;      // [2]
  uint64_t* p_full = s_full + 2;      // [2 tiles][2 key halves]
  uint64_t* o_full = p_full + 4;      // [2]
  uint64_t* q_empty = o_full + 2;     // [1] mode 0: the item's last Q K^T is done
  uint64_t* o_free = q_empty + 1;     // [2] mode 0: the epilogue has read O_w
  uint64_t* drain = o_free + 2;       // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kTmemSlot);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSK; ++s) { mbar_init(&k_full[s], 1); mbar_init(&k_empty[s], 1); }
    for (int s = 0; s < NSV; ++s) { mbar_init(&v_full[s], 1); mbar_init(&v_empty[s], 1); }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&q_full[w], MODE == 0 ? 1 : kRows);  // mode 0: TMA bytes; mode 1: every row's thread
      mbar_init(&o_free[w], 4);
      mbar_init(&s_full[w], 1);
      mbar_init(&p_full[2 * w], 4);
      mbar_init(&p_full[2 * w + 1], 4);
      mbar_init(&o_full[w], 1);
    }
    mbar_init(q_empty, 1);
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    if (MODE == 0) prefetch_tmap(&tmQ);
    if (MODE == 0 && p.anchor_k_on) prefetch_tmap(&tmKA);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  // Registers: the producer/MMA warpgroup (warps 0-3) needs fewer than the softmax
  // warpgroups, which hold a 128-score row each (RegSplit).
  if (warp < 4) {
  setmaxnreg_dec<RegSplit<D>::kCtl>();
  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t kcnt = 0, vcnt = 0;
      bool ok = true;
      // Test hook: CTA 0 issues no first K load, so every role's bounded wait runs out.
      const bool skip_first = blockIdx.x == 0 && (g_debug_flags & kDebugSkipFirstLoad);
      for (int idx = blockIdx.x; idx < p.num_items && ok; idx += gridDim.x) {
        const Item it = decode_item<MODE>(p, idx);
        if (it.skip) continue;
        const int nt = it.a_tiles + it.b_tiles;
        for (int j = 0; j < nt && ok; ++j) {
          const int k0 = tile_key0(it, j);
          int page = p.page_table[(size_t)it.bi * p.max_pages + k0 / p.P];
          if (page < 0 || page >= p.num_pages) { record_error(kDevBadPage); page = 0; }
          const int slot = k0 % p.P;
          {
            const int s = kcnt % NSK;
            ok = mbar_wait(&k_empty[s], ((kcnt / NSK) & 1) ^ 1, kDevTimeoutProducer);
            if (!ok) break;
            uint8_t* dst = smem + S::kK + s * S::kTile;
            if (skip_first && kcnt == 0) {
              // (test hook) no arrival and no load: k_full[0] never completes
            } else if (MODE == 0 && p.anchor_k_on && j < it.a_tiles) {
              mbar_arrive_expect_tx(&k_full[s], S::kTile);
              // The anchor's keys roped at the caller's ids: [B][n-1][Hkv][a][d], block it.part.
#pragma unroll
              for (int h = 0; h < D / 64; ++h)
                tma_load_4d(dst + h * (kKeys * 128), &tmKA, &k_full[s], h * 64, j * kKeys, it.g,
                            it.bi * (p.n - 1) + it.part - 1);
            } else {
              mbar_arrive_expect_tx(&k_full[s], S::kTile);
#pragma unroll
              for (int h = 0; h < D / 64; ++h)
                tma_load_4d(dst + h * (kKeys * 128), &tmK, &k_full[s], h * 64, slot, it.g, page);
            }
            ++kcnt;
          }
          {
            const int s = vcnt % NSV;
            ok = mbar_wait(&v_empty[s], ((vcnt / NSV) & 1) ^ 1, kDevTimeoutProducer);
            if (!ok) break;
            mbar_arrive_expect_tx(&v_full[s], S::kTile);
            uint8_t* dst = smem + S::kV + s * S::kTile;
#pragma unroll
            for (int h = 0; h < D / 64; ++h)
              tma_load_4d(dst + h * (kKeys * 128), &tmV, &v_full[s], h * 64, slot, it.g, page);
            ++vcnt;
          }
        }
      }
      // Drain: every load issued into a stage has landed before the CTA exits.
      for (uint32_t s = 0; s < NSK && s < kcnt; ++s) {
        const uint32_t last = kcnt - 1 - ((kcnt - 1 - s) % NSK);
        mbar_wait(&k_full[s], (last / NSK) & 1, kDevTimeoutProducer);
      }
      for (uint32_t s = 0; s < NSV && s < vcnt; ++s) {
        const uint32_t last = vcnt - 1 - ((vcnt - 1 - s) % NSV);
        mbar_wait(&v_full[s], (last / NSV) & 1, kDevTimeoutProducer);
      }
    }
  } else if (MODE == 0 && warp == 3) {
    // ------------------------------------------------------------------ Q producer (mode 0)
    // The two Q tiles of each item (rows r0 .. r0 + 127 of two query heads, already
    // rotated) by TMA, as soon as the previous item's last Q K^T has completed.
    if (lane == 0) {
      uint32_t qc = 0;
      bool ok = true;
      for (int idx = blockIdx.x; idx < p.num_items && ok; idx += gridDim.x) {
        const Item it = decode_item<MODE>(p, idx);
        if (it.skip) continue;
        if (qc > 0) ok = mbar_wait(q_empty, (qc - 1) & 1, kDevTimeoutProducer);
        if (!ok) break;
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          mbar_arrive_expect_tx(&q_full[w], S::kTile);
#pragma unroll
          for (int h = 0; h < D / 64; ++h)
            tma_load_4d(smem + S::kQ0 + w * S::kTile + h * (kRows * 128), &tmQ, &q_full[w], h * 64,
                        it.g * p.G + 2 * it.hp + w, it.r0 - p.row_off, it.bi);
        }
        ++qc;
      }
      // Drain: the last loads have landed before the CTA exits.
      if (qc > 0) {
        mbar_wait(&q_full[0], (qc - 1) & 1, kDevTimeoutProducer);
        mbar_wait(&q_full[1], (qc - 1) & 1, kDevTimeoutProducer);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = umma_idesc_bf16(kRows, kKeys, 0, 0);
      constexpr uint32_t idesc_pv = umma_idesc_bf16(kRows, D, 0, 1);
      const uint32_t sQ = smem_u32(smem + S::kQ0);
      const uint32_t sK = smem_u32(smem + S::kK);
      const uint32_t sV = smem_u32(smem + S::kV);
      uint32_t kcnt = 0, vcnt = 0, qph = 0, pph[4] = {0, 0, 0, 0};
      bool ok = true;
      bool issued = false;

      // S_w = Q_w K^T: K-major A and B, 128-byte swizzle, 8-row groups 1024 B apart;
      // a 16-element K step is 32 B inside a 64-column atom, atoms are 16 KB apart.
      auto issue_s = [&](int w, int ks) {
        const uint32_t qa = sQ + w * S::kTile;
        const uint32_t kb = sK + ks * S::kTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * (kRows * 128) + (kk % 4) * 32;
          mma_ss(tbase + w * 128, umma_desc_sw128(qa + off, 16, 1024), umma_desc_sw128(kb + off, 16, 1024),
                 idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      // O_w += P_w V: P from TMEM (8 columns per 16 keys); V MN-major (d contiguous),
      // 8 keys of 128 B per swizzle group (SBO 1024 B), 64-column d atoms 16 KB apart (LBO).
      // Issued per 64-key half as soon as the softmax has stored that half of P_w,
      // so the first half's product overlaps the second half's exponentials.
      uint32_t nitem = 0;
      auto issue_pv = [&](int w, int vs, bool acc) -> bool {
        const uint32_t vb = sV + vs * S::kTile;
        // Mode 0: the first product of an item overwrites O_w, which the previous
        // item's epilogue must have read.
        if (MODE == 0 && !acc && nitem > 0 && !mbar_wait(&o_free[w], (nitem - 1) & 1, kDevTimeoutMma)) return false;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if (!mbar_wait(&p_full[2 * w + half], pph[2 * w + half], kDevTimeoutMma)) return false;
          pph[2 * w + half] ^= 1;
          tc_fence_after();
#pragma unroll
          for (int kk = half * 4; kk < half * 4 + 4; ++kk)
            mma_ts(tbase + 256 + w * 128, tbase + w * 128 + kk * 8,
                   umma_desc_sw128(vb + kk * 2048, kKeys * 128, 1024), idesc_pv, (acc || kk > 0) ? 1u : 0u);
        }
        return true;
      };

      for (int idx = blockIdx.x; idx < p.num_items && ok; idx += gridDim.x) {
        const Item it = decode_item<MODE>(p, idx);
        const int nt = it.a_tiles + it.b_tiles;
        if (it.skip || nt == 0) continue;  // padding rows, or a Phase-2 chunk past the sequence
        ok = mbar_wait(&q_full[0], qph, kDevTimeoutMma) && mbar_wait(&q_full[1], qph, kDevTimeoutMma);
        if (!ok) break;
        qph ^= 1;
        tc_fence_after();
        for (int j = 0; j < nt; ++j) {
          const int ks = kcnt % NSK;
          ok = mbar_wait(&k_full[ks], (kcnt / NSK) & 1, kDevTimeoutMma);
          if (!ok) break;
          tc_fence_after();
          int vs = 0;
          if (j > 0) {
            vs = vcnt % NSV;
            ok = mbar_wait(&v_full[vs], (vcnt / NSV) & 1, kDevTimeoutMma) && issue_pv(0, vs, j > 1);
            if (!ok) break;
          }
          issue_s(0, ks);
          issued = true;
          mma_commit(&s_full[0]);
          if (j > 0) {
            ok = issue_pv(1, vs, j > 1);
            if (!ok) break;
            mma_commit(&v_empty[vs]);
            ++vcnt;
          }
          issue_s(1, ks);
          mma_commit(&s_full[1]);
          mma_commit(&k_empty[ks]);
          if (MODE == 0 && j == nt - 1) mma_commit(q_empty);
          ++kcnt;
        }
        if (!ok) break;
        // The last tile's P V products.
        const int vs = vcnt % NSV;
        ok = mbar_wait(&v_full[vs], (vcnt / NSV) & 1, kDevTimeoutMma) && issue_pv(0, vs, nt > 1);
        if (!ok) break;
        mma_commit(&o_full[0]);
        ok = issue_pv(1, vs, nt > 1);
        if (!ok) break;
        mma_commit(&v_empty[vs]);
        ++vcnt;
        mma_commit(&o_full[1]);
        ++nitem;
      }
      if (issued) {
        // Every MMA this thread issued has completed before TMEM is released.
        mma_commit(drain);
        mbar_wait(drain, 0, kDevTimeoutMma);
      }
    }
  }
  } else {
    setmaxnreg_inc<RegSplit<D>::kSoftmax>();
    // ------------------------------------------------------------------ softmax warpgroups
    const int wg = (warp - 4) / 4;
    const int wq = warp % 4;
    const int row = wq * 32 + lane;
    const uint32_t tl = tbase + ((uint32_t)(wq * 32) << 16);
    const uint32_t tS = tl + wg * 128;
    const uint32_t tO = tl + 256 + wg * 128;
    uint8_t* sQ = smem + S::kQ0 + wg * S::kTile;
    uint32_t sph = 0, oph = 0;
    bool ok = true;

    for (int idx = blockIdx.x; idx < p.num_items && ok; idx += gridDim.x) {
      int nt, a_tiles, a_start, a_end, b_start, cache_idx;
      {
        const Item it = decode_item<MODE>(p, idx);
        if (it.skip) continue;
        const RowInfo ri = row_info<MODE>(p, it, wg, row);
        nt = it.a_tiles + it.b_tiles;
        if (MODE == 1 && nt == 0) {
          // A chunk past the sequence's context: an empty partial (O = 0, LSE = -inf),
          // which the merge skips.
          if (ri.valid) {
            const size_t rowoff = (((size_t)it.part * p.B + it.bi) * p.Ntok + ri.tok) * p.Hq + ri.head;
            float4* d4 = reinterpret_cast<float4*>(p.out_f32 + rowoff * D);
#pragma unroll
            for (int e = 0; e < D / 4; ++e) d4[e] = make_float4(0.f, 0.f, 0.f, 0.f);
            p.lse_f32[rowoff] = -INFINITY;
          }
          continue;
        }
        if (MODE == 1) load_q_row<D>(p, it, ri, sQ, row);  // mode 0: Q arrives by TMA
        a_tiles = it.a_tiles;
        a_start = it.a_start;
        a_end = it.a_end;
        b_start = it.b_start;
        cache_idx = ri.cache_idx;
      }
      if (MODE == 1) {
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&q_full[wg]);
      }

      float m = -INFINITY, l = 0.f, lr = 0.f;
      for (int j = 0; j < nt; ++j) {
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[wg], sph, kDevTimeoutSoftmax));
        if (!ok) break;
        sph ^= 1;
        tc_fence_after();
        uint32_t sr[kKeys];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
        tmem_ld_wait();
        // Visible keys of this tile: lo <= key <= hi (the run's range, and causal by
        // cache index).  The second run's tiles start at b_start rounded down to 128.
        int k0, lo, hi;
        if (j < a_tiles) {
          k0 = a_start + j * kKeys;
          lo = a_start;
          hi = min(a_end - 1, cache_idx);
        } else {
          k0 = (b_start & ~(kKeys - 1)) + (j - a_tiles) * kKeys;
          lo = b_start;
          hi = cache_idx;
        }
        if (k0 < lo || k0 + kKeys - 1 > hi) {
          const int clo = lo - k0, chi = hi - k0;  // keys k0 + c with c outside [clo, chi] are not visible
#pragma unroll
          for (int c = 0; c < kKeys; ++c)
            if (c < clo || c > chi) sr[c] = __float_as_uint(-INFINITY);
        }
        // Row max of the raw scores (scale > 0 commutes with max); 4 independent chains.
        float mx[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) mx[e] = fmaxf(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1]));
#pragma unroll
        for (int c = 8; c < kKeys; c += 8)
#pragma unroll
          for (int e = 0; e < 4; ++e)
            mx[e] = fmax3(mx[e], __uint_as_float(sr[c + 2 * e]), __uint_as_float(sr[c + 2 * e + 1]));
        const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        const float m_new = fmaxf(m, mt * p.scale_log2);
        float f = 1.f;
        const bool rescale = m_new > m + kRescaleThreshold;
        if (rescale) {
          f = (l > 0.f) ? ex2_approx(m - m_new) : 1.f;
          m = m_new;
        }
        const float mu = (m == -INFINITY) ? 0.f : m;
        // tcgen05.ld/st are warp-collective (.sync.aligned): the whole warp takes
        // this branch when any of its rows must rescale; the others scale by 1.
        // O_w holds the products of tiles < j only (s_full of tile j is committed
        // after the P V of tile j - 1), so it can be scaled in place; 8 columns at a
        // time, since the 128 scores of the row are live here.
        if (__any_sync(0xffffffffu, f != 1.f)) {
#pragma unroll 1
          for (int c = 0; c < D / 8; ++c) {
            uint32_t o[8];
            tmem_ld8(tO + c * 8, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 8; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
            tmem_st8(tO + c * 8, o);
          }
        }
        // P = 2^(s*scale - m) (exponent arguments two at a time), rounded to bf16 for
        // the P V product; l sums the f32 values (the log-sum-exp needs no bf16
        // rounding in it), two at a time.  Each 64-key half of P goes to TMEM (32
        // columns) and is handed to the MMA warp before the next half is computed.
        const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2);
        const uint64_t nm2 = f2_pack(-mu, -mu);
        uint64_t su2[2] = {0ull, 0ull};
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int cc = half * 32 + c;
            float x0, x1;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[2 * cc]), __uint_as_float(sr[2 * cc + 1])), sc2, nm2), x0, x1);
            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
            pk[c] = pack_bf16x2(p0, p1);
            su2[c & 1] = f2_add(su2[c & 1], f2_pack(p0, p1));
          }
          tmem_st32(tS + half * 32, pk);
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_full[2 * wg + half]);
        }
        float s0, s1, s2, s3;
        f2_unpack(su2[0], s0, s1);
        f2_unpack(su2[1], s2, s3);
        const float rs_u = (s0 + s1) + (s2 + s3);
        // O is normalised by the sum of the bf16-rounded P so that it stays a convex
        // combination of V rows when one key dominates; the rounding that matters
        // there is the largest P's, so its error is added to the f32 sum.
        const float pmax = ex2_approx(fmaf(mt, p.scale_log2, -mu));
        const float rs_r = rs_u + (__bfloat162float(__float2bfloat16_rn(pmax)) - pmax);
        l = l * f + rs_u;
        lr = lr * f + rs_r;
      }
      if (!ok) break;
      ok = __all_sync(0xffffffffu, mbar_wait(&o_full[wg], oph, kDevTimeoutSoftmax));
      if (!ok) break;
      oph ^= 1;
      tc_fence_after();
      const Item it = decode_item<MODE>(p, idx);
      const RowInfo ri = row_info<MODE>(p, it, wg, row);
      const float inv_l = (lr > 0.f) ? 1.f / lr : 0.f;
      if (MODE == 0) {
        bf16* dst = p.out_bf16 + (((size_t)it.bi * p.Lrows + (ri.tok - p.row_off)) * p.Hq + ri.head) * D;
        const bool keep = ri.tok < ctx_len(p, it.bi);  // rows past a shorter sequence are padding
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_ld_wait();
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
          uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
          if (keep) {
#pragma unroll
            for (int e = 0; e < 4; ++e) d4[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
          }
        }
        // O_w is read: the next item's first P V may overwrite it.
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&o_free[wg]);
      } else {
        const size_t rowoff = (((size_t)it.part * p.B + it.bi) * p.Ntok + ri.tok) * p.Hq + ri.head;
        float* dst = p.out_f32 + rowoff * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_ld_wait();
          if (ri.valid) {
            float4* d4 = reinterpret_cast<float4*>(dst + c * 32);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              d4[e] = make_float4(__uint_as_float(o[4 * e]) * inv_l, __uint_as_float(o[4 * e + 1]) * inv_l,
                                  __uint_as_float(o[4 * e + 2]) * inv_l, __uint_as_float(o[4 * e + 3]) * inv_l);
          }
        }
        if (ri.valid) {
          const float lse = (l > 0.f) ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
          p.lse_f32[rowoff] = lse;
        }
      }
      tc_fence_before();
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// Pool [num_pages][Hkv][P][d] bf16 as a 4-D tensor (d innermost); box = 64 x 128 x 1 x 1.
bool make_pool_map(CUtensorMap* map, void* pool, int d, int P, int Hkv, int num_pages) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)P, (cuuint64_t)Hkv, (cuuint64_t)num_pages};
  const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)P * d * 2, (cuuint64_t)Hkv * P * d * 2};
  const cuuint32_t box[4] = {64, (cuuint32_t)kKeys, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, pool, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Rotated queries [B][L][Hq][d] bf16 as a 4-D tensor (d innermost); box = 64 x 1 head x 128 rows x 1.
bool make_q_map(CUtensorMap* map, const void* q, int d, int Hq, int L, int B) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)Hq, (cuuint64_t)L, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)Hq * d * 2, (cuuint64_t)L * Hq * d * 2};
  const cuuint32_t box[4] = {64, 1, (cuuint32_t)kRows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(q), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The anchor's keys [B*(n-1)][Hkv][a][d] bf16 as a 4-D tensor (d innermost); box = 64 x 128 keys x 1 x 1.
bool make_anchor_map(CUtensorMap* map, const void* ka, int d, int a, int Hkv, int nseq) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)a, (cuuint64_t)Hkv, (cuuint64_t)nseq};
  const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)a * d * 2, (cuuint64_t)Hkv * a * d * 2};
  const cuuint32_t box[4] = {64, (cuuint32_t)kKeys, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ka), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int pow2_at_least(int x) {
  int v = 1;
  while (v < x) v <<= 1;
  return v;
}

template <int D, int MODE>
cudaError_t launch_typed(const AttnLaunch& a, const Params& p, const CUtensorMap& mk, const CUtensorMap& mv,
                         const CUtensorMap& mq, const CUtensorMap& mka, cudaStream_t st) {
  constexpr int NSK = (D == 128) ? 2 : 4;
  constexpr int NSV = (D == 128) ? 2 : 4;
  using S = Smem<D, MODE, NSK, NSV>;
  auto kern = star_attn_kernel<D, MODE, NSK, NSV>;
  static std::atomic<unsigned long long> smem_opted_in{0};
  cudaError_t e = opt_in_dynamic_smem(reinterpret_cast<const void*>(kern), S::kBytes, smem_opted_in);
  if (e != cudaSuccess) return e;
  const int grid = std::min(p.num_items, current_device_sm_count());
  if (grid <= 0) return cudaSuccess;
  kern<<<grid, kThreads, S::kBytes, st>>>(mk, mv, mq, mka, p);
  return cudaGetLastError();
}

}  // namespace

int attn_num_parts(const AttnLaunch& a) { return a.n * a.chunks_per_block; }

cudaError_t launch_attention(const AttnLaunch& a, cudaStream_t st, const char** why) {
  Params p;
  memset(&p, 0, sizeof(p));
  p.q = reinterpret_cast<const bf16*>(a.q);
  p.out_bf16 = reinterpret_cast<bf16*>(a.out_bf16);
  p.out_f32 = a.out_f32;
  p.lse_f32 = a.lse_f32;
  p.page_table = a.cache.page_table;
  p.max_pages = a.cache.max_pages;
  p.num_pages = a.cache.num_pages;
  p.P = a.cache.P;
  p.B = a.B;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.G = a.Hq / a.Hkv;
  p.L = a.L;
  p.b = a.b;
  p.n = a.n;
  p.Ntok = a.Ntok;
  p.scale_log2 = a.scale_log2;
  p.blk0 = a.blk0;
  p.nblk = a.nblk ? a.nblk : a.n - a.blk0;
  p.tail_on = a.blk0 + p.nblk == a.n && !a.no_tail;
  p.row_off = a.mode == 0 ? a.blk0 * a.b : 0;
  p.Lrows = a.mode == 0 ? p.nblk * a.b : 0;
  if (a.blk0 < 0 || p.nblk < 1 || a.blk0 + p.nblk > a.n) {
    if (why) *why = "block range outside the context";
    return cudaErrorInvalidValue;
  }
  if (a.mode == 0) {
    p.num_items = a.B * a.Hkv * p.nblk * (a.b / kRows) * (p.G / 2);
  } else {
    p.chunks_per_block = a.chunks_per_block;
    p.chunk_keys = a.b / a.chunks_per_block;
    p.tail_tiles = (a.Ntok + kKeys - 1) / kKeys;
    p.TQ = std::min(pow2_at_least(a.Ntok), kRows);
    p.HT = kRows / p.TQ;
    p.NTT = (a.Ntok + p.TQ - 1) / p.TQ;
    p.NHT = (p.G + p.HT - 1) / p.HT;
    p.npairs = (p.NTT * p.NHT + 1) / 2;
    p.num_items = p.nblk * a.chunks_per_block * a.B * a.Hkv * p.npairs;
  }
  CUtensorMap mk, mv;
  if (!make_pool_map(&mk, a.cache.k_pool, a.d, a.cache.P, a.Hkv, a.cache.num_pages) ||
      !make_pool_map(&mv, a.cache.v_pool, a.d, a.cache.P, a.Hkv, a.cache.num_pages)) {
    if (why) *why = "cuTensorMapEncodeTiled failed for the KV pools";
    return cudaErrorInvalidValue;
  }
  CUtensorMap mq = mk;  // mode 1 stages Q with its own threads; the map is unused there
  if (a.mode == 0 && !make_q_map(&mq, a.q, a.d, a.Hq, p.Lrows, a.B)) {
    if (why) *why = "cuTensorMapEncodeTiled failed for the rotated queries";
    return cudaErrorInvalidValue;
  }
  CUtensorMap mka = mk;  // unused unless the anchor's keys are roped at caller ids
  p.anchor = a.mode == 0 ? a.anchor : 0;
  p.sh = a.shift;
  p.anchor_k_on = (a.mode == 0 && a.anchor_k && a.n > 1) ? 1 : 0;
  if (p.anchor_k_on && !make_anchor_map(&mka, a.anchor_k, a.d, a.anchor, a.Hkv, a.B * (a.n - 1))) {
    if (why) *why = "cuTensorMapEncodeTiled failed for the anchor's keys";
    return cudaErrorInvalidValue;
  }
  if (a.d == 128) {
    return a.mode == 0 ? launch_typed<128, 0>(a, p, mk, mv, mq, mka, st) : launch_typed<128, 1>(a, p, mk, mv, mq, mka, st);
  } else {
    return a.mode == 0 ? launch_typed<64, 0>(a, p, mk, mv, mq, mka, st) : launch_typed<64, 1>(a, p, mk, mv, mq, mka, st);
  }
}

cudaError_t read_and_clear_error_attn(int* code) { return read_and_clear_tu_error(code); }
cudaError_t set_debug_attn(unsigned long long wait_limit_ns, int flags) { return set_tu_debug(wait_limit_ns, flags); }

}  // namespace star
