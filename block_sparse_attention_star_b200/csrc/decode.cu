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
// byte is fetched once for G heads.  The grid is sized to two CTAs per SM, one
// wave.
//
// CTA: warp 8 is the TMA producer (64-key K and V tiles, 128-byte swizzle, a
// 3- or 2-stage ring, no multicast); warps 0-7 compute, per tile:
//   1. QK: thread (key pair kp, dim eighth e) reads 16 dims of keys kp and kp+32
//      (swizzled, conflict-free) and the G query vectors' same 16 dims (shared-
//      memory broadcast), and writes G x 2 partial dot products.
//   2. softmax: warp h owns head h: sums the 8 partials, masks keys past the
//      cache, and updates its running max / sum (online softmax, base 2).
//   3. PV: warp w accumulates keys [8w, 8w+8) into its lanes' 4 dims x G heads.
// At the end the 8 warps' accumulators are reduced and the chunk's normalised
// O and natural-log LSE are written for the merge kernel.
#include "common.cuh"
#include "internal.h"

#include <algorithm>

namespace star {
namespace {

constexpr int kCompute = 256;          // compute threads (8 warps)
constexpr int kThreads = kCompute + 32; // + producer warp
constexpr int kTileKeys = 64;
constexpr int kCtasPerSm = 2;
constexpr int kMaxChunk = 1 << 16;

template <int G>
struct DecCfg {
  static constexpr int NST = (G <= 4) ? 3 : 2;
};

struct DecParams {
  const bf16* q;
  const int32_t* pos;
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
  static constexpr int NST = DecCfg<G>::NST;
  static constexpr int kTile = kTileKeys * D * 2;         // one K or V tile
  static constexpr int kStage = 2 * kTile;                 // K then V
  static constexpr int kQ = NST * kStage;                  // f32 [G][D]
  static constexpr int kPart = kQ + G * D * 4;             // f32 [8][G][64]
  static constexpr int kP = kPart + 8 * G * kTileKeys * 4; // f32 [64][G]
  static constexpr int kStat = kP + kTileKeys * G * 4;     // f32 alpha[G], m[G], l[G]
  static constexpr int kBar = ((kStat + 3 * G * 4) + 7) / 8 * 8;
  static constexpr int kEnd = kBar + 2 * NST * 8;
  static constexpr int kBytes = kEnd + 1024;
  static_assert(8 * G * D * 4 <= NST * kStage, "final reduction must fit in the stage buffers");
};

// Byte offset of element (key, d) in a swizzled 64-key tile: 64-element d halves
// are separate [64 keys][128 B] boxes; 16-byte chunks are XOR-permuted by key % 8.
__device__ __forceinline__ int tile_off(int key, int d) {
  const int half = d >> 6, e = d & 63;
  return half * (kTileKeys * 128) + key * 128 + ((((e >> 3) ^ (key & 7)) << 4) | ((e & 7) << 1));
}

__device__ __forceinline__ void bar_compute() { asm volatile("bar.sync 1, %0;" ::"n"(kCompute) : "memory"); }

// Barrier over the compute warps that also returns whether `v` holds in all of them,
// so every warp takes the same give-up decision.
__device__ __forceinline__ bool bar_compute_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(kCompute)
      : "memory");
  return r != 0;
}

template <int D, int G>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ DecParams p) {
  using S = DecSmem<D, G>;
  constexpr int NST = S::NST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* qs = reinterpret_cast<float*>(smem + S::kQ);
  float* part = reinterpret_cast<float*>(smem + S::kPart);
  float* ps = reinterpret_cast<float*>(smem + S::kP);
  float* stat = reinterpret_cast<float*>(smem + S::kStat);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBar);
  uint64_t* empty = full + NST;

  const int c = blockIdx.x % p.nchunks;
  const int g = (blockIdx.x / p.nchunks) % p.Hkv;
  const int bi = blockIdx.x / (p.nchunks * p.Hkv);
  const int k_begin = c * p.chunk;
  const int k_end = min(k_begin + p.chunk, p.n_keys);
  const int ntiles = (k_end - k_begin + kTileKeys - 1) / kTileKeys;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    fence_barrier_init();
  }
  // q of the G heads: RoPE at the token's position (float64 rotation, one bf16
  // rounding, as the cache keys), then scaled by log2(e)/sqrt(d).
  const int tpos = p.pos[bi];
  for (int e = threadIdx.x; e < G * (D / 2); e += kThreads) {
    const int h = e / (D / 2), j = e % (D / 2);
    const bf16* qr = p.q + ((size_t)bi * p.Hq + g * G + h) * D;
    const double x1 = __bfloat162float(qr[j]), x2 = __bfloat162float(qr[j + D / 2]);
    double cs, sn;
    rope_sincos(tpos, p.inv_freq[j], cs, sn);
    qs[h * D + j] = __bfloat162float(__double2bfloat16(x1 * cs - x2 * sn)) * p.scale_log2;
    qs[h * D + j + D / 2] = __bfloat162float(__double2bfloat16(x2 * cs + x1 * sn)) * p.scale_log2;
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
    constexpr int DPT = D / 8;                  // QK: dims per thread (one eighth of d)
    constexpr int DPL = D / 32;                 // PV: dims per lane
    const int t = threadIdx.x;
    const int kp = t & 31, e8 = t >> 5;         // QK: key pair, dim eighth (= warp)
    float m_run = -INFINITY, l_run = 0.f;       // warp h < G: stats of head h
    float acc[G][DPL];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int i = 0; i < DPL; ++i) acc[h][i] = 0.f;
    bool ok = true;

    for (int tt = 0; tt < ntiles; ++tt) {
      const int s = tt % NST;
      const bool arrived = mbar_wait(&full[s], (tt / NST) & 1, kDevTimeoutSoftmax);
      const uint8_t* kt = smem + s * S::kStage;
      const uint8_t* vt = kt + S::kTile;

      // 1. partial dot products over dims [DPT e8, DPT e8 + DPT) for keys kp, kp + 32
      {
        float d0[G], d1[G];
#pragma unroll
        for (int h = 0; h < G; ++h) d0[h] = d1[h] = 0.f;
#pragma unroll
        for (int ch = 0; ch < DPT / 8; ++ch) {
          const int dbase = DPT * e8 + 8 * ch;
          const uint4 ka = *reinterpret_cast<const uint4*>(kt + tile_off(kp, dbase));
          const uint4 kb = *reinterpret_cast<const uint4*>(kt + tile_off(kp + 32, dbase));
          const uint32_t* wa = reinterpret_cast<const uint32_t*>(&ka);
          const uint32_t* wb = reinterpret_cast<const uint32_t*>(&kb);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float4 q0 = *reinterpret_cast<const float4*>(qs + h * D + dbase);
            const float4 q1 = *reinterpret_cast<const float4*>(qs + h * D + dbase + 4);
            const float qv[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 fa = unpack_bf16x2(wa[i]);
              const float2 fb = unpack_bf16x2(wb[i]);
              d0[h] = fmaf(qv[2 * i], fa.x, fmaf(qv[2 * i + 1], fa.y, d0[h]));
              d1[h] = fmaf(qv[2 * i], fb.x, fmaf(qv[2 * i + 1], fb.y, d1[h]));
            }
          }
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
          part[(e8 * G + h) * kTileKeys + kp] = d0[h];
          part[(e8 * G + h) * kTileKeys + kp + 32] = d1[h];
        }
      }
      ok = bar_compute_all(arrived);
      if (!ok) break;

      // 2. online softmax, warp h < G owns head h (keys lane and lane + 32)
      if (warp < G) {
        const int h = warp;
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          s0 += part[(e * G + h) * kTileKeys + lane];
          s1 += part[(e * G + h) * kTileKeys + lane + 32];
        }
        const int kg = k_begin + tt * kTileKeys;
        if (kg + lane >= k_end) s0 = -INFINITY;
        if (kg + lane + 32 >= k_end) s1 = -INFINITY;
        float mt = fmaxf(s0, s1);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
        const float m_new = fmaxf(m_run, mt);   // the tile's first key is always valid
        const float alpha = ex2_approx(m_run - m_new);
        const float p0 = ex2_approx(s0 - m_new), p1 = ex2_approx(s1 - m_new);
        float ls = p0 + p1;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, off);
        l_run = l_run * alpha + ls;
        m_run = m_new;
        ps[lane * G + h] = p0;
        ps[(lane + 32) * G + h] = p1;
        if (lane == 0) stat[h] = alpha;
      }
      bar_compute();

      // 3. P V: warp w takes keys [8w, 8w + 8); lane owns dims [DPL lane, DPL lane + DPL)
      {
        float al[G];
#pragma unroll
        for (int h = 0; h < G; ++h) al[h] = stat[h];
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
          for (int i = 0; i < DPL; ++i) acc[h][i] *= al[h];
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int key = 8 * warp + kk;
          float vf[DPL];
          if constexpr (DPL == 4) {
            const uint2 vv = *reinterpret_cast<const uint2*>(vt + tile_off(key, 4 * lane));
            const float2 v01 = unpack_bf16x2(vv.x), v23 = unpack_bf16x2(vv.y);
            vf[0] = v01.x; vf[1] = v01.y; vf[2] = v23.x; vf[3] = v23.y;
          } else {
            const float2 v01 = unpack_bf16x2(*reinterpret_cast<const uint32_t*>(vt + tile_off(key, 2 * lane)));
            vf[0] = v01.x; vf[1] = v01.y;
          }
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float pw = ps[key * G + h];
#pragma unroll
            for (int i = 0; i < DPL; ++i) acc[h][i] = fmaf(pw, vf[i], acc[h][i]);
          }
        }
      }
      bar_compute();
      if (t == 0) mbar_arrive(&empty[s]);
    }

    // Final reduction over the 8 warps (reusing the stage buffers: all consumed).
    if (ok) {
      float* red = reinterpret_cast<float*>(smem);   // [8][G][D]
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int i = 0; i < DPL; ++i) red[(warp * G + h) * D + DPL * lane + i] = acc[h][i];
      if (warp < G && lane == 0) {
        stat[G + warp] = m_run;
        stat[2 * G + warp] = l_run;
      }
      bar_compute();
      const size_t rows = (size_t)p.B * p.Hq;
      for (int idx = t; idx < G * D; idx += kCompute) {
        const int h = idx / D;
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) sum += red[(w * G + h) * D + (idx % D)];
        const float l = stat[2 * G + h];
        const size_t row = (size_t)bi * p.Hq + g * G + h;
        p.o_ws[((size_t)c * rows + row) * D + (idx % D)] = (l > 0.f) ? sum / l : 0.f;
        if (idx % D == 0)
          p.lse_ws[(size_t)c * rows + row] = (l > 0.f) ? (stat[G + h] + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      }
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

int decode_num_chunks(int n_keys, int chunk) { return (n_keys + chunk - 1) / chunk; }

// Chunks per (sequence, KV head) so that the grid is one wave of two CTAs per SM;
// the chunk is a multiple of the 64-key tile.
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

cudaError_t read_and_clear_error_decode(int* code) { return read_and_clear_tu_error(code); }

cudaError_t launch_decode(const DecodeLaunch& a, cudaStream_t st) {
  DecParams p;
  p.q = reinterpret_cast<const bf16*>(a.q);
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
