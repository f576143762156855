// Star Attention decode: one generated token attends to the whole cache
// ("Star Attention: Efficient LLM Inference over Long Sequences", abstract:
// response tokens attend to all prior cached tokens; "Star Attention 完全拆解(一)",
// "Phase 2: 局部注意力与本地统计量": each block yields a local output and its
// softmax statistic, merged exactly in "组装全局结果").
//
// HBM-bound: a step reads every cached K and V byte once.  The cache is cut into
// chunks (a finer partition than blocks; the merge is associative, so chunk
// partials merge to the same result as per-block partials).  One CTA per
// (chunk, KV head, sequence) serves all G query heads of the group, so each K/V
// byte is fetched once for G heads.  The grid is one wave of kCtasPerSm CTAs per SM.
//
// The CTA that owns the last chunk of a (sequence, KV head) first appends the new
// token: RoPE(k) (float64 rotation, one bf16 rounding, like star_kv_append) and v
// go to cache slot n_keys - 1, made visible to its own TMA loads by a proxy fence.
//
// CTA: warp 8 is the TMA producer (64-key K and V tiles, 128-byte swizzle, an
// NST-stage ring, no multicast); warps 0-7 compute.  Warp w owns keys
// [8w, 8w + 8) of every tile and keeps its own online softmax (running max m and
// sum l per head, base 2), so there is no CTA barrier per tile:
//   QK: lane = (key kk = lane / 4, quarter = lane % 4); it dots its quarter of
//       the key with the same quarter of the G query vectors (shared-memory
//       broadcast from a padded layout); two shuffles finish the dot products.
//   softmax: max and sum over the warp's 8 keys by shuffles; P goes to a small
//       per-warp shared buffer.
//   PV: lane owns d/32 dims of the G outputs and accumulates the 8 keys.
// At the end the 8 warps' (m, l, O) are combined and the chunk's normalised O and
// natural-log LSE are written for the merge kernel.
#include "common.cuh"
#include "internal.h"

#include <algorithm>

namespace star {
namespace {

constexpr int kCompute = 256;            // compute threads (8 warps)
constexpr int kThreads = kCompute + 32;  // + producer warp
constexpr int kTileKeys = 64;
constexpr int kMaxChunk = 1 << 16;
constexpr int kCtasPerSm = 2;
constexpr int kStages = 3;

struct DecParams {
  const bf16* q;       // [B][Hq][D]
  const bf16* k_new;   // [B][Hkv][D]: the token appended at slot n_keys - 1
  const bf16* v_new;
  bf16* kpool;
  bf16* vpool;
  const int32_t* pos;  // [B]
  const int32_t* page_table;
  float* o_ws;
  float* lse_ws;
  int max_pages, num_pages, P;
  int B, Hq, Hkv, n_keys, chunk, nchunks;
  float scale_log2;
  double inv_freq[kMaxHalfDim];
};

template <int D, int G>
struct DecSmem {
  static constexpr int NST = kStages;
  static constexpr int QPAD = D / 4 + 4;                  // floats per (head, quarter) row
  static constexpr int kTile = kTileKeys * D * 2;         // one K or V tile
  static constexpr int kStage = 2 * kTile;                // K then V
  static constexpr int kQ = NST * kStage;                 // f32 [G][4][QPAD]
  static constexpr int kP = kQ + G * 4 * QPAD * 4;        // f32 [8 warps][8 keys][G]
  static constexpr int kBar = (kP + 8 * 8 * G * 4 + 7) / 8 * 8;
  static constexpr int kEnd = kBar + 2 * NST * 8;
  static constexpr int kBytes = kEnd + 1024;
  static_assert(8 * G * (D + 2) * 4 <= NST * kStage, "final combine must fit in the stage buffers");
};

// Byte offset of element (key, d) in a swizzled 64-key tile: 64-element d halves
// are separate [64 keys][128 B] boxes; 16-byte chunks are XOR-permuted by key % 8.
__device__ __forceinline__ int tile_off(int key, int d) {
  const int half = d >> 6, e = d & 63;
  return half * (kTileKeys * 128) + key * 128 + ((((e >> 3) ^ (key & 7)) << 4) | ((e & 7) << 1));
}

__device__ __forceinline__ void bar_compute() { asm volatile("bar.sync 1, %0;" ::"n"(kCompute) : "memory"); }

__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

template <int D, int G>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ DecParams p) {
  using S = DecSmem<D, G>;
  constexpr int NST = S::NST;
  constexpr int QPAD = S::QPAD;
  constexpr int DQ = D / 4;    // dims per quarter (QK)
  constexpr int DPL = D / 32;  // dims per lane (PV)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* qs = reinterpret_cast<float*>(smem + S::kQ);
  float* ps_all = reinterpret_cast<float*>(smem + S::kP);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBar);
  uint64_t* empty = full + NST;

  const int c = blockIdx.x % p.nchunks;
  const int g = (blockIdx.x / p.nchunks) % p.Hkv;
  const int bi = blockIdx.x / (p.nchunks * p.Hkv);
  const int k_begin = c * p.chunk;
  const int k_end = min(k_begin + p.chunk, p.n_keys);
  const int ntiles = (k_end - k_begin + kTileKeys - 1) / kTileKeys;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int tpos = p.pos[bi];

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 8);
    }
    fence_barrier_init();
  }
  // The owner of the last chunk appends the new token (head g) before any load.
  if (c == p.nchunks - 1) {
    const int slot_abs = p.n_keys - 1;
    const int page = p.page_table[(size_t)bi * p.max_pages + slot_abs / p.P];
    if (page < 0 || page >= p.num_pages) {
      if (threadIdx.x == 0) record_error(kDevBadPage);
    } else {
      const size_t dst = (((size_t)page * p.Hkv + g) * p.P + (slot_abs % p.P)) * D;
      const size_t src = ((size_t)bi * p.Hkv + g) * D;
      for (int e = threadIdx.x; e < D / 4; e += kThreads) {
        // pairs (j, j + 1) of the first half with the same pairs of the second half, j = 2e
        const uint32_t a = *reinterpret_cast<const uint32_t*>(p.k_new + src + 2 * e);
        const uint32_t b = *reinterpret_cast<const uint32_t*>(p.k_new + src + D / 2 + 2 * e);
        double cs[2], sn[2];
        rope_sincos(tpos, p.inv_freq[2 * e], cs[0], sn[0]);
        rope_sincos(tpos, p.inv_freq[2 * e + 1], cs[1], sn[1]);
        uint32_t lo, hi;
        rope_rotate2(a, b, cs, sn, lo, hi);
        *reinterpret_cast<uint32_t*>(p.kpool + dst + 2 * e) = lo;
        *reinterpret_cast<uint32_t*>(p.kpool + dst + D / 2 + 2 * e) = hi;
      }
      for (int e = threadIdx.x; e < D / 2; e += kThreads)
        *reinterpret_cast<uint32_t*>(p.vpool + dst + 2 * e) =
            *reinterpret_cast<const uint32_t*>(p.v_new + src + 2 * e);
      fence_proxy_async_global();
    }
  }
  // q of the G heads: RoPE at the token's position (float64 rotation, one bf16
  // rounding, as the cache keys), scaled by log2(e)/sqrt(d), stored per quarter
  // with padding so that the four quarters' broadcasts fall in different banks.
  for (int e = threadIdx.x; e < G * (D / 2); e += kThreads) {
    const int h = e / (D / 2), j = e % (D / 2);
    const bf16* qr = p.q + ((size_t)bi * p.Hq + g * G + h) * D;
    const double x1 = __bfloat162float(qr[j]), x2 = __bfloat162float(qr[j + D / 2]);
    double cs, sn;
    rope_sincos(tpos, p.inv_freq[j], cs, sn);
    const int d1 = j, d2 = j + D / 2;
    qs[(h * 4 + d1 / DQ) * QPAD + d1 % DQ] = __bfloat162float(__double2bfloat16(x1 * cs - x2 * sn)) * p.scale_log2;
    qs[(h * 4 + d2 / DQ) * QPAD + d2 % DQ] = __bfloat162float(__double2bfloat16(x2 * cs + x1 * sn)) * p.scale_log2;
  }
  __syncthreads();

  if (warp == 8) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      bool ok = true;
      for (int t = 0; t < ntiles && ok; ++t) {
        const int s = t % NST;
        ok = mbar_wait(&empty[s], ((t / NST) & 1) ^ 1, kDevTimeoutProducer);
        if (!ok) break;
        const int k0 = k_begin + t * kTileKeys;
        int page = p.page_table[(size_t)bi * p.max_pages + k0 / p.P];
        if (page < 0 || page >= p.num_pages) {
          record_error(kDevBadPage);
          page = 0;
        }
        const int slot = k0 % p.P;
        mbar_arrive_expect_tx(&full[s], 2 * S::kTile);
        uint8_t* dk = smem + s * S::kStage;
        uint8_t* dv = dk + S::kTile;
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
          tma_load_4d(dk + h * (kTileKeys * 128), &tmK, &full[s], h * 64, slot, g, page);
          tma_load_4d(dv + h * (kTileKeys * 128), &tmV, &full[s], h * 64, slot, g, page);
        }
      }
      // Every load issued has landed before the CTA may exit.
      for (int s = 0; s < NST && s < ntiles; ++s) {
        const int last = ntiles - 1 - ((ntiles - 1 - s) % NST);
        mbar_wait(&full[s], (last / NST) & 1, kDevTimeoutProducer);
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- compute
    const int kk = lane >> 2, qd = lane & 3;  // QK: key within the warp's 8, quarter of d
    float* ps = ps_all + warp * 8 * G;         // this warp's P: [8 keys][G]
    float m_run[G], l_run[G], acc[G][DPL];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m_run[h] = -INFINITY;
      l_run[h] = 0.f;
#pragma unroll
      for (int i = 0; i < DPL; ++i) acc[h][i] = 0.f;
    }
    bool ok = true;

    for (int tt = 0; tt < ntiles; ++tt) {
      const int s = tt % NST;
      ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (tt / NST) & 1, kDevTimeoutSoftmax));
      if (!ok) break;
      const uint8_t* kt = smem + s * S::kStage;
      const uint8_t* vt = kt + S::kTile;
      const int key = 8 * warp + kk;

      // QK over this lane's quarter, then across the key's four lanes.
      float sc[G];
#pragma unroll
      for (int h = 0; h < G; ++h) sc[h] = 0.f;
#pragma unroll
      for (int i = 0; i < DQ / 8; ++i) {
        const uint4 kv = *reinterpret_cast<const uint4*>(kt + tile_off(key, qd * DQ + 8 * i));
        const uint32_t* w = reinterpret_cast<const uint32_t*>(&kv);
        float kf[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = unpack_bf16x2(w[e]);
          kf[2 * e] = f.x;
          kf[2 * e + 1] = f.y;
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float* qrow = qs + (h * 4 + qd) * QPAD + 8 * i;
          const float4 q0 = *reinterpret_cast<const float4*>(qrow);
          const float4 q1 = *reinterpret_cast<const float4*>(qrow + 4);
          float a = sc[h];
          a = fmaf(q0.x, kf[0], a);
          a = fmaf(q0.y, kf[1], a);
          a = fmaf(q0.z, kf[2], a);
          a = fmaf(q0.w, kf[3], a);
          a = fmaf(q1.x, kf[4], a);
          a = fmaf(q1.y, kf[5], a);
          a = fmaf(q1.z, kf[6], a);
          a = fmaf(q1.w, kf[7], a);
          sc[h] = a;
        }
      }
      const bool valid = (k_begin + tt * kTileKeys + key) < k_end;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        sc[h] += __shfl_xor_sync(0xffffffffu, sc[h], 1);
        sc[h] += __shfl_xor_sync(0xffffffffu, sc[h], 2);
        if (!valid) sc[h] = -INFINITY;
      }
      // Online softmax over the warp's 8 keys (lanes 4kk..4kk+3 hold key kk).
      float al[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float mt = sc[h];
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 4));
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 8));
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
        const float m_new = fmaxf(m_run[h], mt);
        const float mu = (m_new == -INFINITY) ? 0.f : m_new;
        al[h] = ex2_approx(m_run[h] - mu);
        const float pv = ex2_approx(sc[h] - mu);
        float ls = pv;
        ls += __shfl_xor_sync(0xffffffffu, ls, 4);
        ls += __shfl_xor_sync(0xffffffffu, ls, 8);
        ls += __shfl_xor_sync(0xffffffffu, ls, 16);
        l_run[h] = l_run[h] * al[h] + ls;
        m_run[h] = m_new;
        if (qd == 0) ps[kk * G + h] = pv;
      }
      __syncwarp();
      // P V: lane owns dims [DPL lane, DPL lane + DPL) of the G outputs.
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int i = 0; i < DPL; ++i) acc[h][i] *= al[h];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int vkey = 8 * warp + j;
        float vf[DPL];
        if constexpr (DPL == 4) {
          const uint2 vv = *reinterpret_cast<const uint2*>(vt + tile_off(vkey, 4 * lane));
          const float2 v01 = unpack_bf16x2(vv.x), v23 = unpack_bf16x2(vv.y);
          vf[0] = v01.x;
          vf[1] = v01.y;
          vf[2] = v23.x;
          vf[3] = v23.y;
        } else {
          const float2 v01 = unpack_bf16x2(*reinterpret_cast<const uint32_t*>(vt + tile_off(vkey, 2 * lane)));
          vf[0] = v01.x;
          vf[1] = v01.y;
        }
        float pj[G];
        if constexpr (G % 4 == 0) {
#pragma unroll
          for (int h = 0; h < G; h += 4) {
            const float4 p4 = *reinterpret_cast<const float4*>(ps + j * G + h);
            pj[h] = p4.x;
            pj[h + 1] = p4.y;
            pj[h + 2] = p4.z;
            pj[h + 3] = p4.w;
          }
        } else {
#pragma unroll
          for (int h = 0; h < G; ++h) pj[h] = ps[j * G + h];
        }
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
          for (int i = 0; i < DPL; ++i) acc[h][i] = fmaf(pj[h], vf[i], acc[h][i]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }

    // Combine the 8 warps (reusing the stage buffers once every tile is consumed).
    // A warp that gave up a wait still joins both barriers, so none is left waiting.
    bar_compute();
    float* red = reinterpret_cast<float*>(smem);  // [8][G][D] accumulators
    float* st = red + 8 * G * D;                  // [8][G][2]: m, l
#pragma unroll
    for (int h = 0; h < G; ++h) {
#pragma unroll
      for (int i = 0; i < DPL; ++i) red[(warp * G + h) * D + DPL * lane + i] = acc[h][i];
      if (lane == 0) {
        st[(warp * G + h) * 2] = m_run[h];
        st[(warp * G + h) * 2 + 1] = l_run[h];
      }
    }
    bar_compute();
    const size_t rows = (size_t)p.B * p.Hq;
    for (int idx = threadIdx.x; idx < G * D; idx += kCompute) {
      const int h = idx / D, dd = idx % D;
      float mstar = -INFINITY;
#pragma unroll
      for (int w = 0; w < 8; ++w) mstar = fmaxf(mstar, st[(w * G + h) * 2]);
      float sum = 0.f, l = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const float mw = st[(w * G + h) * 2];
        const float f = (mw == -INFINITY) ? 0.f : ex2_approx(mw - mstar);
        sum += f * red[(w * G + h) * D + dd];
        l += f * st[(w * G + h) * 2 + 1];
      }
      const size_t row = (size_t)bi * p.Hq + g * G + h;
      p.o_ws[((size_t)c * rows + row) * D + dd] = (l > 0.f) ? sum / l : 0.f;
      if (dd == 0)
        p.lse_ws[(size_t)c * rows + row] = (l > 0.f) ? (mstar + __log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
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
cudaError_t launch_dg(const DecParams& p, const CUtensorMap& mk, const CUtensorMap& mv, cudaStream_t st) {
  using S = DecSmem<D, G>;
  auto kern = decode_kernel<D, G>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kBytes);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  kern<<<p.nchunks * p.Hkv * p.B, kThreads, S::kBytes, st>>>(mk, mv, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t read_and_clear_error_decode(int* code) { return read_and_clear_tu_error(code); }

int decode_num_chunks(int n_keys, int chunk) { return (n_keys + chunk - 1) / chunk; }

// Chunks per (sequence, KV head) so that the grid is one wave of kCtasPerSm CTAs
// per SM; the chunk is a multiple of the 64-key tile.
int decode_pick_chunk(int B, int Hkv, int G, int n_keys, int num_sms) {
  (void)G;
  long long per_head = (long long)kCtasPerSm * num_sms / ((long long)B * Hkv);
  if (per_head < 1) per_head = 1;
  long long chunk = (n_keys + per_head - 1) / per_head;
  chunk = (chunk + kTileKeys - 1) / kTileKeys * kTileKeys;
  chunk = std::max<long long>(kTileKeys, std::min<long long>(kMaxChunk, chunk));
  return (int)chunk;
}

size_t decode_smem_bytes(int d, int G, int chunk) {
  (void)chunk;
  if (d == 128) {
    switch (G) {
      case 1: return DecSmem<128, 1>::kBytes;
      case 2: return DecSmem<128, 2>::kBytes;
      case 4: return DecSmem<128, 4>::kBytes;
      default: return DecSmem<128, 8>::kBytes;
    }
  }
  switch (G) {
    case 1: return DecSmem<64, 1>::kBytes;
    case 2: return DecSmem<64, 2>::kBytes;
    case 4: return DecSmem<64, 4>::kBytes;
    default: return DecSmem<64, 8>::kBytes;
  }
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
  p.nchunks = decode_num_chunks(a.n_keys, a.chunk);
  p.scale_log2 = a.scale_log2;
  for (int j = 0; j < kMaxHalfDim; ++j) p.inv_freq[j] = j < a.d / 2 ? a.rope.inv_freq[j] : 0.0;
  CUtensorMap mk, mv;
  if (!make_tile_map(&mk, a.cache.k_pool, a.d, a.cache.P, a.Hkv, a.cache.num_pages) ||
      !make_tile_map(&mv, a.cache.v_pool, a.d, a.cache.P, a.Hkv, a.cache.num_pages))
    return cudaErrorInvalidValue;
  const int G = a.Hq / a.Hkv;
#define STAR_DEC_CASE(DD, GG) \
  if (a.d == DD && G == GG) return launch_dg<DD, GG>(p, mk, mv, st);
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
