// Star Attention decode: one generated token per sequence attends to the whole
// cache ("Star Attention: Efficient LLM Inference over Long Sequences", abstract:
// response tokens attend to all prior cached tokens; "Star Attention 完全拆解(一)",
// "Phase 2: 局部注意力与本地统计量": each block yields a local output and its
// softmax statistic, merged exactly in "组装全局结果").
//
// HBM-bound: a step reads every cached K and V byte once.  The cache of each
// (sequence, KV head) is cut into chunks of whole 128-key tiles (a finer partition
// than blocks; the merge is associative, so chunk partials merge to the same result
// as per-block partials).  A work item is one (sequence, KV head, chunk); a
// persistent CTA per SM takes items round-robin and streams their tiles through
// one TMA ring, so the loads never stop at item boundaries.
//
// The G query heads of a GQA group against one 128-key tile are a dense product
// (G x d times d x 128).  It runs on the tensor core in transposed form, so that
// the 128 keys fill the UMMA M dimension and the heads, padded to 16, are N:
//   S^T [128 keys x 16]  = K_tile [128 x d] . Q_g^T             (K-major A and B)
//   O^T [d x 16]         = V_tile^T [d x 128 keys] . P^T        (MN-major A, K-major B)
// K and V tiles land by TMA in the Phase-1 layout ([key][64 d] boxes, 128-byte
// swizzle), which is exactly the K-major A operand of S^T and the MN-major A
// operand of O^T.  Each tile's O^T goes to a fresh TMEM accumulator and is added
// into registers with the online-softmax rescale, so no TMEM value is rewritten.
//
// Softmax threads own one key of S^T and one dimension of O^T each (TMEM lane =
// thread), so a tile costs them a few dozen instructions: the kernel streams at
// HBM rate instead of being bound by instruction issue, as a CUDA-core dot-product
// formulation of the same step is (about 80 instructions per key and head group).
//
// The CTA owning the last chunk of a (sequence, KV head) appends the new token:
// RoPE(k) (float64 rotation, one bf16 rounding, like star_kv_append) and v go to
// cache slot n_keys - 1, made visible to its own TMA loads by a proxy fence and an
// mbarrier that the producer waits on before the tile holding that slot.
//
// CTA (256 threads, one per SM):
//   warp 0     TMA producer (K and V rings, loaded by this CTA only)
//   warp 1     TMEM allocation and MMA issuer
//   warps 2-7  prologue (append, q) while warp 0 already streams K and V
//   warps 4-7  then softmax and O accumulation: thread = TMEM lane 32 (w - 4) + lane
#include "common.cuh"
#include "internal.h"

#include <algorithm>

namespace star {
namespace {

constexpr int kThreads = 256;
constexpr int kTileKeys = 128;           // UMMA M of S^T, K of O^T
constexpr int kStages = 3;               // K/V ring depth
constexpr int kMaxItems = 8;             // items per CTA per launch (q of each stays in shared memory)
constexpr int kProWarps = 6;             // warps 2-7 run the prologue (append, q)
constexpr int kProThreads = 32 * kProWarps;
constexpr uint32_t kTmemCols = 64;       // S^T: [0,16) [16,32); O^T: [32,48) [48,64)
constexpr uint32_t kIdescQK = umma_idesc_bf16(128, 16, 0, 0);
constexpr uint32_t kIdescPV = umma_idesc_bf16(128, 16, 1, 0);

struct DecParams {
  const bf16* q;       // [B][Hq][D]
  const bf16* k_new;   // [B][Hkv][D]: the token appended at slot n_keys - 1
  const bf16* v_new;
  bf16* kpool;
  bf16* vpool;
  const int32_t* pos;  // [B]
  const int32_t* page_table;
  float* o_ws;         // [nchunks][B*Hq][D]
  float* lse_ws;       // [nchunks][B*Hq]
  int max_pages, num_pages, P;
  int B, Hq, Hkv, n_keys, chunk, nchunks;
  int k_lo;                  // first key of the range (0, or a shard's first block's first key)
  int append;                // the range holds the new token's slot n_keys - 1 (it is appended here)
  int item_base, num_items;  // this launch: items [item_base, num_items)
  float scale_log2;
  SeqShift sh;               // sequence bi has n_keys + delta[bi] keys (sh.on = 0: all n_keys)
  // sh.on: the item space lists every sequence's non-empty chunks first (sequence bi's
  // at [item_off[bi], item_off[bi+1]), head-major, chunk fastest), then the empty chunk
  // slots past the shorter sequences ([item_off[B] + empty_off[bi], ...)), so that the
  // round-robin assignment spreads the real work evenly over the CTAs.
  int item_off[kMaxVarB + 1];
  int empty_off[kMaxVarB + 1];
  double inv_freq[kMaxHalfDim];
};

template <int D>
struct DecSmem {
  static constexpr int kTile = kTileKeys * D * 2;    // D/64 boxes of [128 keys][128 B]
  // The V ring comes first: for D = 64 the M = 128 view of a V tile reads the
  // 16 KB after it (rows 64-127 of O^T, never used), which must be shared memory.
  static constexpr int kV = 0;
  static constexpr int kK = kV + kStages * kTile;
  static constexpr int kQItem = (D / 64) * 1024;      // D/64 atoms of [8 heads][128 B]
  static constexpr int kQ = kK + kStages * kTile;
  static constexpr int kP = kQ + kMaxItems * kQItem;   // 2 buffers x 2 atoms (keys 0-63, 64-127)
  static constexpr int kPad = kP + 2 * 2048;          // read by the N = 16 view of the last P atom
  static constexpr int kXch = kPad + 1024;            // f32 [2][4 warps][8 heads]: warp maxima
  static constexpr int kRed = kXch + 2 * 4 * 8 * 4;   // f32 [4 warps][8 heads][2]: sums
  static constexpr int kTab = kRed + 4 * 8 * 2 * 4;   // f64 (cos, sin) [kMaxItems][D/2]: RoPE of the token
  static constexpr int kTabOf = kTab + kMaxItems * (D / 2) * 16;  // int [kMaxItems]: table used by each item
  static constexpr int kBar = kTabOf + kMaxItems * 4;
  static constexpr int kNumBars = 4 * kStages + 6 * 2 + 3;
  static constexpr int kSlot = kBar + kNumBars * 8;
  static constexpr int kBytes = kSlot + 16 + 1024;    // + alignment slack
  static_assert(kBytes <= 227 * 1024, "decode shared memory");
};

struct DecItem {
  int bi, g, c, k_begin, k_end, ntiles;
  int n_keys;  // keys of this sequence
  int last;    // the chunk holds the sequence's last key (the new token's slot)
};

// The last sequence s in [0, B) with off[s] <= x (off is non-decreasing, off[0] = 0 <= x).
__device__ __forceinline__ int seq_of(const int* off, int B, int x) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= x) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ DecItem dec_item(const DecParams& p, int idx) {
  DecItem it;
  if (!p.sh.on) {
    it.c = idx % p.nchunks;
    it.g = (idx / p.nchunks) % p.Hkv;
    it.bi = idx / (p.nchunks * p.Hkv);
  } else if (idx < p.item_off[p.B]) {
    it.bi = seq_of(p.item_off, p.B, idx);
    const int w = idx - p.item_off[it.bi];
    const int nc = (p.item_off[it.bi + 1] - p.item_off[it.bi]) / p.Hkv;
    it.g = w / nc;
    it.c = w - it.g * nc;
  } else {
    const int e = idx - p.item_off[p.B];
    it.bi = seq_of(p.empty_off, p.B, e);
    const int w = e - p.empty_off[it.bi];
    const int ne = (p.empty_off[it.bi + 1] - p.empty_off[it.bi]) / p.Hkv;
    it.g = w / ne;
    it.c = p.nchunks - ne + (w - it.g * ne);
  }
  it.n_keys = p.n_keys + (p.sh.on ? p.sh.delta[it.bi] : 0);
  it.k_begin = p.k_lo + it.c * p.chunk;
  it.k_end = min(it.k_begin + p.chunk, it.n_keys);
  // A chunk past a shorter sequence's keys is empty (0 tiles): its partial is O = 0, LSE = -inf.
  it.ntiles = it.k_end > it.k_begin ? (it.k_end - it.k_begin + kTileKeys - 1) / kTileKeys : 0;
  it.last = p.append && (it.c == (it.n_keys - 1 - p.k_lo) / p.chunk);
  return it;
}

// Byte offset of (row, element e) in a K-major 128-byte-swizzle atom of 8 rows x 64 bf16.
__device__ __forceinline__ int sw128(int row, int e) {
  return row * 128 + ((((e >> 3) ^ (row & 7)) << 4) | ((e & 7) << 1));
}

// tcgen05.ld, 32 lanes x N columns of 32 bit (N = 1, 2, 4, 8).
template <int N>
__device__ __forceinline__ void tmem_ld_n(uint32_t taddr, uint32_t (&r)[N]);
template <>
__device__ __forceinline__ void tmem_ld_n<1>(uint32_t taddr, uint32_t (&r)[1]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r[0]) : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld_n<2>(uint32_t taddr, uint32_t (&r)[2]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld_n<4>(uint32_t taddr, uint32_t (&r)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld_n<8>(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}

__device__ __forceinline__ float warp_max(float x) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

template <int D, int G>
__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ DecParams p) {
  using S = DecSmem<D>;
  constexpr int NST = kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
  uint64_t* k_full = bars;
  uint64_t* k_empty = bars + NST;
  uint64_t* v_full = bars + 2 * NST;
  uint64_t* v_empty = bars + 3 * NST;
  uint64_t* s_full = bars + 4 * NST;  // [2] each
  uint64_t* s_empty = s_full + 2;
  uint64_t* p_full = s_full + 4;
  uint64_t* o_full = s_full + 6;
  uint64_t* o_empty = s_full + 8;
  uint64_t* x_bar = s_full + 10;
  uint64_t* red_bar = s_full + 12;
  uint64_t* drain = s_full + 13;
  uint64_t* pro_done = s_full + 14;  // warps 2-7 have appended the token and staged q
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kSlot);
  float* xch = reinterpret_cast<float*>(smem + S::kXch);
  float* red = reinterpret_cast<float*>(smem + S::kRed);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int first = p.item_base + blockIdx.x;
  const int n_my = min(kMaxItems, (p.num_items - first + (int)gridDim.x - 1) / (int)gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_empty[b], 4);
      mbar_init(&p_full[b], 4);
      mbar_init(&o_full[b], 1);
      mbar_init(&o_empty[b], 4);
      mbar_init(&x_bar[b], 4);
    }
    mbar_init(red_bar, 4);
    mbar_init(drain, 1);
    mbar_init(pro_done, kProWarps);
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  // q and P operands: the padding rows (heads G..15) are zeros.
  for (int i = threadIdx.x; i < (S::kXch - S::kQ) / 16; i += kThreads)
    reinterpret_cast<uint4*>(smem + S::kQ)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  // Everything above touches only this CTA's on-chip state, so it overlaps the
  // previous kernel's tail; global memory is read and written only after it ends.
  griddep_wait();
  griddep_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  // Warps 2-7 append the token and stage q (below) while the producer already
  // streams K and V; the producer waits for the append only before the tile that
  // holds the new slot, and the MMA warp waits for q before its first product.
  if (warp >= 2) {
    const int pt = threadIdx.x - 64;
    // The token's rotation angles, once per run of items of the same sequence (the
    // append and the G query heads of every such item use the same D/2 angles);
    // tab_of[ii] is the item whose table item ii uses.
    double2* tab = reinterpret_cast<double2*>(smem + S::kTab);
    int* tab_of = reinterpret_cast<int*>(smem + S::kTabOf);
    {
      int prev_bi = -1, cur = 0;
      for (int ii = 0; ii < n_my; ++ii) {
        const int bi = dec_item(p, first + ii * gridDim.x).bi;
        if (bi != prev_bi) {
          prev_bi = bi;
          cur = ii;
          const int tpos = p.pos[bi];
          for (int j = pt; j < D / 2; j += kProThreads) {
            double c, sn;
            rope_sincos(tpos, p.inv_freq[j], c, sn);
            tab[ii * (D / 2) + j] = make_double2(c, sn);
          }
        }
        if (pt == 0) tab_of[ii] = cur;
      }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kProThreads) : "memory");

    // Append the new token (head g) for each item that holds its sequence's last key.
    for (int ii = 0; ii < n_my; ++ii) {
      const DecItem it = dec_item(p, first + ii * gridDim.x);
      if (!it.last) continue;
      const double2* ang = tab + tab_of[ii] * (D / 2);
      const int slot_abs = it.n_keys - 1;
      const int page = p.page_table[(size_t)it.bi * p.max_pages + slot_abs / p.P];
      if (page < 0 || page >= p.num_pages) {
        if (pt == 0) record_error(kDevBadPage);
        continue;
      }
      const size_t dst = (((size_t)page * p.Hkv + it.g) * p.P + (slot_abs % p.P)) * D;
      const size_t src = ((size_t)it.bi * p.Hkv + it.g) * D;
      for (int e = pt; e < D / 4; e += kProThreads) {
        // pairs (j, j + 1) of the first half with the same pairs of the second half, j = 2e
        const uint32_t a = *reinterpret_cast<const uint32_t*>(p.k_new + src + 2 * e);
        const uint32_t b = *reinterpret_cast<const uint32_t*>(p.k_new + src + D / 2 + 2 * e);
        const double2 a0 = ang[2 * e], a1 = ang[2 * e + 1];
        const double cs[2] = {a0.x, a1.x}, sn[2] = {a0.y, a1.y};
        uint32_t lo, hi;
        rope_rotate2(a, b, cs, sn, lo, hi);
        *reinterpret_cast<uint32_t*>(p.kpool + dst + 2 * e) = lo;
        *reinterpret_cast<uint32_t*>(p.kpool + dst + D / 2 + 2 * e) = hi;
      }
      for (int e = pt; e < D / 2; e += kProThreads)
        *reinterpret_cast<uint32_t*>(p.vpool + dst + 2 * e) = *reinterpret_cast<const uint32_t*>(p.v_new + src + 2 * e);
    }

    // q of the G heads of every item: RoPE at the token's position (float64 rotation,
    // one bf16 rounding, as the cache keys), as the K-major B operand [head][d].  A
    // unit is 8 rotation pairs of one head: two 16-byte loads, two 16-byte stores.
    constexpr int kUnits = G * (D / 16);
    for (int u = pt; u < n_my * kUnits; u += kProThreads) {
      const int ii = u / kUnits, h = (u % kUnits) / (D / 16), c = u % (D / 16);
      const DecItem it = dec_item(p, first + ii * gridDim.x);
      const bf16* qr = p.q + ((size_t)it.bi * p.Hq + it.g * G + h) * D;
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(qr + 8 * c));
      const uint4 b = __ldg(reinterpret_cast<const uint4*>(qr + D / 2 + 8 * c));
      const double2* ang = tab + tab_of[ii] * (D / 2) + 8 * c;
      const uint32_t* aw = reinterpret_cast<const uint32_t*>(&a);
      const uint32_t* bw = reinterpret_cast<const uint32_t*>(&b);
      uint32_t lo[4], hi[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const double2 a0 = ang[2 * e], a1 = ang[2 * e + 1];
        const double cs[2] = {a0.x, a1.x}, sn[2] = {a0.y, a1.y};
        rope_rotate2(aw[e], bw[e], cs, sn, lo[e], hi[e]);
      }
      uint8_t* qs = smem + S::kQ + ii * S::kQItem;
      const int d1 = 8 * c, d2 = D / 2 + 8 * c;
      *reinterpret_cast<uint4*>(qs + (d1 / 64) * 1024 + sw128(h, d1 % 64)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      *reinterpret_cast<uint4*>(qs + (d2 / 64) * 1024 + sw128(h, d2 % 64)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    }
    // The appended K/V (global) and q (shared) are read next by the async proxy (TMA, MMA).
    fence_proxy_async_global();
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(pro_done);
  }

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      uint32_t kc = 0;
      bool ok = true;
      // Test hook: CTA 0 issues no first K load, so every role's bounded wait runs out.
      const bool skip_first = blockIdx.x == 0 && (g_debug_flags & kDebugSkipFirstLoad);
      for (int ii = 0; ii < n_my && ok; ++ii) {
        const DecItem it = dec_item(p, first + ii * gridDim.x);
        for (int t = 0; t < it.ntiles && ok; ++t, ++kc) {
          const int k0 = it.k_begin + t * kTileKeys;
          // The tile holding the new token's slot is loaded after the append.
          if (it.last && t == it.ntiles - 1 && !mbar_wait(pro_done, 0, kDevTimeoutProducer)) {
            ok = false;
            break;
          }
          int page = p.page_table[(size_t)it.bi * p.max_pages + k0 / p.P];
          if (page < 0 || page >= p.num_pages) {
            record_error(kDevBadPage);
            page = 0;
          }
          const int slot = k0 % p.P;
          const int s = kc % NST;
          const uint32_t ph = ((kc / NST) & 1) ^ 1;
          ok = mbar_wait(&k_empty[s], ph, kDevTimeoutProducer);
          if (!ok) break;
          if (!(skip_first && kc == 0)) {  // (test hook) no arrival and no load: k_full[0] never completes
            mbar_arrive_expect_tx(&k_full[s], S::kTile);
#pragma unroll
            for (int h = 0; h < D / 64; ++h)
              tma_load_4d(smem + S::kK + s * S::kTile + h * (kTileKeys * 128), &tmK, &k_full[s], h * 64, slot, it.g,
                          page);
          }
          ok = mbar_wait(&v_empty[s], ph, kDevTimeoutProducer);
          if (!ok) break;
          mbar_arrive_expect_tx(&v_full[s], S::kTile);
#pragma unroll
          for (int h = 0; h < D / 64; ++h)
            tma_load_4d(smem + S::kV + s * S::kTile + h * (kTileKeys * 128), &tmV, &v_full[s], h * 64, slot, it.g,
                        page);
        }
      }
      // Every load issued has landed before the CTA may exit.
      for (uint32_t s = 0; s < (uint32_t)NST && s < kc; ++s) {
        const uint32_t last = kc - 1 - ((kc - 1 - s) % NST);
        mbar_wait(&k_full[s], (last / NST) & 1, kDevTimeoutProducer);
        mbar_wait(&v_full[s], (last / NST) & 1, kDevTimeoutProducer);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t sK = smem_u32(smem + S::kK), sV = smem_u32(smem + S::kV);
      const uint32_t sQ = smem_u32(smem + S::kQ), sP = smem_u32(smem + S::kP);
      bool issued = false;
      // O^T_t = V_t^T P_t^T: V MN-major (d atoms 16 KB apart, 8-key groups 1 KB apart,
      // 16 keys = 2 KB per K step); P K-major (64-key atoms 1 KB apart).
      auto issue_pv = [&](uint32_t t) -> bool {
        const int s = t % NST, b = t & 1;
        if (!mbar_wait(&v_full[s], (t / NST) & 1, kDevTimeoutMma)) return false;
        if (!mbar_wait(&p_full[b], (t >> 1) & 1, kDevTimeoutMma)) return false;
        if (t >= 2 && !mbar_wait(&o_empty[b], ((t >> 1) & 1) ^ 1, kDevTimeoutMma)) return false;
        tc_fence_after();
        const uint32_t va = sV + s * S::kTile, pb = sP + b * 2048;
#pragma unroll
        for (int kk = 0; kk < kTileKeys / 16; ++kk)
          mma_ss(tbase + 32 + 16 * b, umma_desc_sw128(va + kk * 2048, kTileKeys * 128, 1024),
                 umma_desc_sw128(pb + (kk / 4) * 1024 + (kk % 4) * 32, 16, 1024), kIdescPV, kk > 0 ? 1u : 0u);
        mma_commit(&o_full[b]);
        mma_commit(&v_empty[s]);
        return true;
      };
      uint32_t j = 0;
      bool ok = mbar_wait(pro_done, 0, kDevTimeoutMma);  // q of every item is staged
      for (int ii = 0; ii < n_my && ok; ++ii) {
        const DecItem it = dec_item(p, first + ii * gridDim.x);
        const uint32_t qa = sQ + ii * S::kQItem;
        for (int t = 0; t < it.ntiles; ++t, ++j) {
          const int s = j % NST, b = j & 1;
          ok = mbar_wait(&k_full[s], (j / NST) & 1, kDevTimeoutMma);
          if (ok && j >= 2) ok = mbar_wait(&s_empty[b], ((j >> 1) & 1) ^ 1, kDevTimeoutMma);
          if (!ok) break;
          tc_fence_after();
          // S^T_j = K_j Q^T: K-major, 8-row groups 1 KB apart, 16-element K step = 32 B
          // inside a 64-element atom; K atoms 16 KB apart, q atoms 1 KB apart.
          const uint32_t ka = sK + s * S::kTile;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(tbase + 16 * b, umma_desc_sw128(ka + (kk / 4) * (kTileKeys * 128) + (kk % 4) * 32, 16, 1024),
                   umma_desc_sw128(qa + (kk / 4) * 1024 + (kk % 4) * 32, 16, 1024), kIdescQK, kk > 0 ? 1u : 0u);
          issued = true;
          mma_commit(&s_full[b]);
          mma_commit(&k_empty[s]);
          if (j >= 1) {
            ok = issue_pv(j - 1);
            if (!ok) break;
          }
        }
      }
      if (ok && j >= 1) issue_pv(j - 1);
      if (issued) {
        // Every MMA this thread issued has completed before TMEM is released.
        mma_commit(drain);
        mbar_wait(drain, 0, kDevTimeoutMma);
      }
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- softmax + O
    const int wi = warp - 4;
    const uint32_t tl = tbase + ((uint32_t)(wi * 32) << 16);
    const int kt = wi * 32 + lane;  // key of the tile (S^T lane) and dimension (O^T lane)
    uint8_t* sP = smem + S::kP;
    const size_t rows = (size_t)p.B * p.Hq;
    uint32_t j = 0;
    bool ok = true;
    float o[G], al_prev[G];

    // O_run = O_run * alpha_t + O^T_t for tile t (lane kt = dimension kt).
    auto acc_o = [&](uint32_t t, const float (&al)[G]) -> bool {
      const int b = t & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&o_full[b], (t >> 1) & 1, kDevTimeoutSoftmax))) return false;
      tc_fence_after();
      uint32_t r[G];
      tmem_ld_n<G>(tl + 32 + 16 * b, r);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_empty[b]);
#pragma unroll
      for (int h = 0; h < G; ++h) o[h] = fmaf(o[h], al[h], __uint_as_float(r[h]));
      return true;
    };

    uint32_t nred = 0;  // items that took the row-sum barrier
    for (int ii = 0; ii < n_my && ok; ++ii) {
      const DecItem it = dec_item(p, first + ii * gridDim.x);
      if (it.ntiles == 0) {
        // A chunk past this sequence's keys: an empty partial (O = 0, LSE = -inf), which
        // the merge skips; no tile of it is loaded or multiplied.
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const size_t row = (size_t)it.bi * p.Hq + it.g * G + h;
          if (kt < D) p.o_ws[((size_t)it.c * rows + row) * D + kt] = 0.f;
          if (kt == h) p.lse_ws[(size_t)it.c * rows + row] = -INFINITY;
        }
        continue;
      }
      float m_run[G], lu[G], lr[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        m_run[h] = -INFINITY;
        lu[h] = 0.f;
        lr[h] = 0.f;
        o[h] = 0.f;
        al_prev[h] = 0.f;
      }
      for (int t = 0; t < it.ntiles; ++t, ++j) {
        const int b = j & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[b], (j >> 1) & 1, kDevTimeoutSoftmax));
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[G];
        tmem_ld_n<G>(tl + 16 * b, sr);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[b]);
        // Scores in base 2; keys past the chunk's end are masked.
        const bool valid = it.k_begin + t * kTileKeys + kt < it.k_end;
        float x[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          x[h] = valid ? __uint_as_float(sr[h]) * p.scale_log2 : -INFINITY;
          const float wm = warp_max(x[h]);
          if (lane == 0) xch[(b * 4 + wi) * 8 + h] = wm;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&x_bar[b]);
        ok = __all_sync(0xffffffffu, mbar_wait(&x_bar[b], (j >> 1) & 1, kDevTimeoutSoftmax));
        if (!ok) break;
        // Tile max over the 4 warps; every tile has a valid key, so m_new is finite.
        float al[G];
        uint8_t* pt = sP + b * 2048 + (kt / 64) * 1024;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float* xw = xch + b * 32 + h;
          const float tm = fmaxf(fmaxf(xw[0], xw[8]), fmaxf(xw[16], xw[24]));
          const float m_new = fmaxf(m_run[h], tm);
          al[h] = ex2_approx(m_run[h] - m_new);  // 0 on the first tile (m_run = -inf)
          m_run[h] = m_new;
          const float pv = ex2_approx(x[h] - m_new);
          const bf16 pb = __float2bfloat16_rn(pv);
          // lu: f32 sum for the log-sum-exp; lr: sum of the bf16 values the product uses.
          lu[h] = fmaf(lu[h], al[h], pv);
          lr[h] = fmaf(lr[h], al[h], __bfloat162float(pb));
          *reinterpret_cast<bf16*>(pt + sw128(h, kt % 64)) = pb;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[b]);
        if (t > 0) {
          ok = acc_o(j - 1, al_prev);
          if (!ok) break;
        }
#pragma unroll
        for (int h = 0; h < G; ++h) al_prev[h] = al[h];
      }
      if (!ok) break;
      ok = acc_o(j - 1, al_prev);
      if (!ok) break;
      // Sums over the 128 keys of the tile lanes (thread partials), then the 4 warps.
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float su = lu[h], sr = lr[h];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          su += __shfl_xor_sync(0xffffffffu, su, off);
          sr += __shfl_xor_sync(0xffffffffu, sr, off);
        }
        if (lane == 0) {
          red[(wi * 8 + h) * 2] = su;
          red[(wi * 8 + h) * 2 + 1] = sr;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(red_bar);
      ok = __all_sync(0xffffffffu, mbar_wait(red_bar, nred & 1, kDevTimeoutSoftmax));
      ++nred;
      if (!ok) break;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float Lu = 0.f, Lr = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          Lu += red[(w * 8 + h) * 2];
          Lr += red[(w * 8 + h) * 2 + 1];
        }
        const size_t row = (size_t)it.bi * p.Hq + it.g * G + h;
        if (kt < D) p.o_ws[((size_t)it.c * rows + row) * D + kt] = o[h] / Lr;
        if (kt == h) p.lse_ws[(size_t)it.c * rows + row] = (m_run[h] + __log2f(Lu)) * 0.69314718055994531f;
      }
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

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool make_tile_map(CUtensorMap* map, void* pool, int d, int P, int Hkv, int num_pages) {
  static EncodeTiledFn enc = nullptr;
  if (!enc) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    enc = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)P, (cuuint64_t)Hkv, (cuuint64_t)num_pages};
  const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)P * d * 2, (cuuint64_t)Hkv * P * d * 2};
  const cuuint32_t box[4] = {64, (cuuint32_t)kTileKeys, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, pool, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int G>
cudaError_t launch_dg(DecParams p, const CUtensorMap& mk, const CUtensorMap& mv, int total_items, cudaStream_t st) {
  using S = DecSmem<D>;
  auto kern = decode_kernel<D, G>;
  static std::atomic<unsigned long long> smem_opted_in{0};
  cudaError_t e0 = opt_in_dynamic_smem(reinterpret_cast<const void*>(kern), S::kBytes, smem_opted_in);
  if (e0 != cudaSuccess) return e0;
  const int grid = std::min(total_items, current_device_sm_count());
  // Each launch covers at most kMaxItems items per CTA.
  for (int base = 0; base < total_items; base += grid * kMaxItems) {
    p.item_base = base;
    p.num_items = std::min(total_items, base + grid * kMaxItems);
    cudaError_t e = launch_pdl(kern, std::min(grid, p.num_items - base), kThreads, S::kBytes, st, mk, mv, p);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t read_and_clear_error_decode(int* code) { return read_and_clear_tu_error(code); }
cudaError_t set_debug_decode(unsigned long long wait_limit_ns, int flags) { return set_tu_debug(wait_limit_ns, flags); }

int decode_num_chunks(int n_keys, int chunk) { return (n_keys + chunk - 1) / chunk; }

// Per-sequence key counts: the chunk (at least min_chunk keys, a multiple of 128) that
// minimises the tiles of the busiest CTA over the non-empty items, with the same quarter
// tile of overhead per item as the uniform choice.
int decode_pick_chunk_var(int B, int Hkv, const int* n_keys_of, int min_chunk, int num_sms) {
  long long tmax = 1;
  for (int s = 0; s < B; ++s) tmax = std::max<long long>(tmax, (n_keys_of[s] + kTileKeys - 1) / kTileKeys);
  const long long ct_min = std::max(1, min_chunk / kTileKeys);
  long long best_ct = std::max(ct_min, tmax), best_cost = -1;
  for (long long ct = ct_min; ct <= tmax; ++ct) {
    long long items = 0;
    for (int s = 0; s < B; ++s) items += (long long)Hkv * ((n_keys_of[s] + ct * kTileKeys - 1) / (ct * kTileKeys));
    const long long ctas = std::min<long long>(items, num_sms);
    const long long per = (items + ctas - 1) / ctas;
    const long long cost = 4 * per * ct + per;
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best_ct = ct;
    }
  }
  return (int)(best_ct * kTileKeys);
}

// Keys per chunk (a multiple of the 128-key tile) for caches of up to n_keys keys:
// the chunk count that minimises the tiles of the busiest CTA, counting each item
// a quarter tile of overhead.
int decode_pick_chunk(int B, int Hkv, int G, int n_keys, int num_sms) {
  (void)G;
  const long long tiles = std::max(1, (n_keys + kTileKeys - 1) / kTileKeys);
  const long long bh = (long long)B * Hkv;
  long long best_ct = tiles, best_cost = -1;
  const long long nc_max = std::min<long long>(tiles, std::max<long long>(1, (long long)kMaxItems * num_sms / bh));
  for (long long nc = 1; nc <= nc_max; ++nc) {
    const long long ct = (tiles + nc - 1) / nc;
    const long long nce = (tiles + ct - 1) / ct;
    const long long items = bh * nce;
    const long long ctas = std::min<long long>(items, num_sms);
    const long long per = (items + ctas - 1) / ctas;
    const long long cost = 4 * per * ct + per;
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best_ct = ct;
    }
  }
  return (int)(best_ct * kTileKeys);
}

cudaError_t launch_decode(const DecodeLaunch& a, cudaStream_t st) {
  DecParams p;
  p.q = reinterpret_cast<const bf16*>(a.q);
  p.k_new = reinterpret_cast<const bf16*>(a.k_new);
  p.v_new = reinterpret_cast<const bf16*>(a.v_new);
  p.kpool = reinterpret_cast<bf16*>(a.cache.k_pool);
  p.vpool = reinterpret_cast<bf16*>(a.cache.v_pool);
  p.pos = a.pos;
  p.page_table = a.cache.page_table;
  p.o_ws = a.o_ws;
  p.lse_ws = a.lse_ws;
  p.max_pages = a.cache.max_pages;
  p.num_pages = a.cache.num_pages;
  p.P = a.cache.P;
  p.B = a.B;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.n_keys = a.n_keys;
  p.chunk = a.chunk;
  p.k_lo = a.k_lo;
  p.append = a.append;
  if (a.k_lo < 0 || a.k_lo % kTileKeys != 0 || a.k_lo >= a.n_keys || (a.k_lo > 0 && a.shift.on))
    return cudaErrorInvalidValue;
  p.nchunks = decode_num_chunks(a.n_keys - a.k_lo, a.chunk);
  p.item_base = 0;
  p.num_items = 0;
  p.scale_log2 = a.scale_log2;
  p.sh = a.shift;
  for (int j = 0; j < kMaxHalfDim; ++j) p.inv_freq[j] = j < a.d / 2 ? a.rope.inv_freq[j] : 0.0;
  if (a.chunk <= 0 || a.chunk % kTileKeys != 0 || a.cache.P % kTileKeys != 0) return cudaErrorInvalidValue;
  p.item_off[0] = p.empty_off[0] = 0;
  if (p.sh.on) {
    if (a.B > kMaxVarB) return cudaErrorInvalidValue;
    for (int s = 0; s < a.B; ++s) {
      const int ks = a.n_keys + p.sh.delta[s];
      if (ks < 1 || ks > a.n_keys) return cudaErrorInvalidValue;
      const int nc = decode_num_chunks(ks, a.chunk);
      p.item_off[s + 1] = p.item_off[s] + a.Hkv * nc;
      p.empty_off[s + 1] = p.empty_off[s] + a.Hkv * (p.nchunks - nc);
    }
  }
  CUtensorMap mk, mv;
  if (!make_tile_map(&mk, a.cache.k_pool, a.d, a.cache.P, a.Hkv, a.cache.num_pages) ||
      !make_tile_map(&mv, a.cache.v_pool, a.d, a.cache.P, a.Hkv, a.cache.num_pages))
    return cudaErrorInvalidValue;
  const int G = a.Hq / a.Hkv;
  const int total = p.nchunks * a.Hkv * a.B;
#define STAR_DEC_CASE(DD, GG) \
  if (a.d == DD && G == GG) return launch_dg<DD, GG>(p, mk, mv, total, st);
  STAR_DEC_CASE(128, 1)
  STAR_DEC_CASE(128, 2)
  STAR_DEC_CASE(128, 4)
  STAR_DEC_CASE(128, 8)
  STAR_DEC_CASE(64, 1)
  STAR_DEC_CASE(64, 2)
  STAR_DEC_CASE(64, 4)
  STAR_DEC_CASE(64, 8)
#undef STAR_DEC_CASE
  return cudaErrorInvalidValue;
}

}  // namespace star
