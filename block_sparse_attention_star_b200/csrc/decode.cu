// Star Attention decode: one generated token attends to the whole cache
// ("Star Attention: Efficient LLM Inference over Long Sequences", abstract:
// response tokens attend to all prior cached tokens; "Star Attention 完全拆解(一)",
// "Phase 2: 局部注意力与本地统计量": each block yields a local output and its
// softmax statistic, merged exactly in "组装全局结果").
//
// The cache is cut into chunks that never straddle a block (chunk | b is not
// required: chunks are a finer partition and the merge is associative, so the
// per-chunk partials merge to the same result as per-block partials).  One CTA
// per (chunk, KV head, sequence) computes the chunk's (O, LSE) for the G query
// heads of the group: every 16-byte K/V load serves all G heads, which is what
// makes this HBM-bound step read the cache exactly once.
//
//   1. q of the G heads: RoPE at the token's position, rounded to bf16, scaled
//      by log2(e)/sqrt(d), kept in shared memory.
//   2. scores: d/8 lanes share one key row (16 B each), dot products reduced by
//      warp shuffles; written to shared memory.
//   3. per-head max / exp2 / sum over the chunk (two-pass softmax, exact).
//   4. P V with the same load pattern; lanes holding the same d-slice reduce by
//      shuffles, warps through shared memory.
#include "common.cuh"
#include "internal.h"

#include <algorithm>

namespace star {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kUnroll = 4;
constexpr int kMaxChunk = 2048;

struct DecParams {
  const bf16* q;
  const int32_t* pos;
  const bf16* kpool;
  const bf16* vpool;
  const int32_t* page_table;
  float* o_ws;
  float* lse_ws;
  int max_pages, num_pages, P;
  int B, Hq, Hkv, n_keys, chunk;
  float scale_log2;
  double inv_freq[kMaxHalfDim];
};

template <int D>
__device__ __forceinline__ const bf16* key_row(const DecParams& p, const bf16* pool, int bi, int g, int kidx) {
  int page = p.page_table[(size_t)bi * p.max_pages + kidx / p.P];
  page = min(max(page, 0), p.num_pages - 1);
  return pool + (((size_t)page * p.Hkv + g) * p.P + (kidx % p.P)) * D;
}

template <int D, int G>
__global__ void __launch_bounds__(kThreads) decode_kernel(const __grid_constant__ DecParams p) {
  constexpr int LPK = D / 8;        // lanes per key row
  constexpr int KPW = 32 / LPK;     // keys per warp step
  extern __shared__ float sm[];
  float* qs = sm;                       // [G][D]
  float* red = qs + G * D;              // [kWarps][G][D]
  float* stat = red + kWarps * G * D;   // m[G], l[G]
  float* sc = stat + 2 * G;             // [G][chunk]

  const int c = blockIdx.x, g = blockIdx.y, bi = blockIdx.z;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int k_begin = c * p.chunk;
  const int nk = min(p.chunk, p.n_keys - k_begin);
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

  const int sub = lane / LPK, part = lane % LPK;
  {
    float qreg[G][8];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < 8; ++e) qreg[h][e] = qs[h * D + part * 8 + e];
    for (int base = warp * KPW; base < nk; base += kWarps * KPW * kUnroll) {
      uint4 kv[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int key = base + u * kWarps * KPW + sub;
        kv[u] = make_uint4(0, 0, 0, 0);
        if (key < nk) kv[u] = __ldg(reinterpret_cast<const uint4*>(key_row<D>(p, p.kpool, bi, g, k_begin + key) + part * 8));
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int key = base + u * kWarps * KPW + sub;
        const uint32_t* w = reinterpret_cast<const uint32_t*>(&kv[u]);
        float kf[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = unpack_bf16x2(w[e]);
          kf[2 * e] = f.x;
          kf[2 * e + 1] = f.y;
        }
        float dot[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float s = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) s = fmaf(qreg[h][e], kf[e], s);
          dot[h] = s;
        }
#pragma unroll
        for (int off = LPK / 2; off > 0; off >>= 1)
#pragma unroll
          for (int h = 0; h < G; ++h) dot[h] += __shfl_xor_sync(0xffffffffu, dot[h], off);
        if (part == 0 && key < nk) {
#pragma unroll
          for (int h = 0; h < G; ++h) sc[h * p.chunk + key] = dot[h];
        }
      }
    }
  }
  __syncthreads();

  if (warp < G) {
    const int h = warp;
    float m = -INFINITY;
    for (int k = lane; k < nk; k += 32) m = fmaxf(m, sc[h * p.chunk + k]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float l = 0.f;
    for (int k = lane; k < nk; k += 32) {
      const float e = ex2_approx(sc[h * p.chunk + k] - m);
      sc[h * p.chunk + k] = e;
      l += e;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    if (lane == 0) {
      stat[h] = m;
      stat[G + h] = l;
    }
  }
  __syncthreads();

  float acc[G][8];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[h][e] = 0.f;
  for (int base = warp * KPW; base < nk; base += kWarps * KPW * kUnroll) {
    uint4 vv[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int key = base + u * kWarps * KPW + sub;
      vv[u] = make_uint4(0, 0, 0, 0);
      if (key < nk) vv[u] = __ldg(reinterpret_cast<const uint4*>(key_row<D>(p, p.vpool, bi, g, k_begin + key) + part * 8));
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int key = base + u * kWarps * KPW + sub;
      if (key >= nk) continue;
      const uint32_t* w = reinterpret_cast<const uint32_t*>(&vv[u]);
      float vf[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = unpack_bf16x2(w[e]);
        vf[2 * e] = f.x;
        vf[2 * e + 1] = f.y;
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float pw = sc[h * p.chunk + key];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[h][e] = fmaf(pw, vf[e], acc[h][e]);
      }
    }
  }
#pragma unroll
  for (int off = LPK; off < 32; off <<= 1)
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[h][e] += __shfl_xor_sync(0xffffffffu, acc[h][e], off);
  if (sub == 0) {
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < 8; ++e) red[(warp * G + h) * D + part * 8 + e] = acc[h][e];
  }
  __syncthreads();

  const size_t rows = (size_t)p.B * p.Hq;
  for (int idx = threadIdx.x; idx < G * D; idx += kThreads) {
    const int h = idx / D;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s += red[w * G * D + idx];
    const float l = stat[G + h];
    const size_t row = (size_t)bi * p.Hq + g * G + h;
    p.o_ws[((size_t)c * rows + row) * D + (idx % D)] = (l > 0.f) ? s / l : 0.f;
    if (idx % D == 0)
      p.lse_ws[(size_t)c * rows + row] = (l > 0.f) ? (stat[h] + __log2f(l)) * 0.69314718055994531f : -INFINITY;
  }
}

template <int D, int G>
cudaError_t launch_dg(const DecParams& p, int nchunks, cudaStream_t st) {
  const size_t smem = decode_smem_bytes(D, G, p.chunk);
  auto kern = decode_kernel<D, G>;
  static size_t attr = 0;
  if (smem > attr) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr = smem;
  }
  dim3 grid(nchunks, p.Hkv, p.B);
  kern<<<grid, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

int decode_num_chunks(int n_keys, int chunk) { return (n_keys + chunk - 1) / chunk; }

int decode_pick_chunk(int B, int Hkv, int G, int n_keys, int num_sms) {
  (void)G;
  const long long target = 4LL * num_sms;
  long long per_head = (target + (long long)B * Hkv - 1) / ((long long)B * Hkv);
  if (per_head < 1) per_head = 1;
  long long chunk = (n_keys + per_head - 1) / per_head;
  chunk = (chunk + 63) / 64 * 64;
  chunk = std::max<long long>(64, std::min<long long>(kMaxChunk, chunk));
  return (int)chunk;
}

size_t decode_smem_bytes(int d, int G, int chunk) {
  return sizeof(float) * ((size_t)G * d + (size_t)kWarps * G * d + 2 * G + (size_t)G * chunk);
}

cudaError_t launch_decode(const DecodeLaunch& a, cudaStream_t st) {
  DecParams p;
  p.q = reinterpret_cast<const bf16*>(a.q);
  p.pos = a.pos;
  p.kpool = reinterpret_cast<const bf16*>(a.cache.k_pool);
  p.vpool = reinterpret_cast<const bf16*>(a.cache.v_pool);
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
  p.scale_log2 = a.scale_log2;
  for (int j = 0; j < kMaxHalfDim; ++j) p.inv_freq[j] = j < a.d / 2 ? a.rope.inv_freq[j] : 0.0;
  const int nchunks = decode_num_chunks(a.n_keys, a.chunk);
  const int G = a.Hq / a.Hkv;
#define STAR_DEC_CASE(DD, GG) \
  if (a.d == DD && G == GG) return launch_dg<DD, GG>(p, nchunks, st);
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
