// Exact merge of attention partials (O_i, LSE_i) into global attention
// ("Star Attention 完全拆解(一)", "组装全局结果": s_global = sum_h s_h and
// A_global = sum_h (s_h / s_global) A_h; "数值稳定性": carried out on
// log-sum-exp values in float32, then cast to the query dtype).
//
// With m = max_i LSE_i over the partials whose LSE is finite,
//   LSE = m + log(sum_i exp(LSE_i - m)),   O = sum_i exp(LSE_i - LSE) O_i.
// A partial with a non-finite LSE (an empty block: -inf) contributes nothing;
// a row with no finite partial gives O = 0, LSE = -inf.
//
// One warp per output row; each lane owns d/32 consecutive columns (one
// 16-byte load per partial at d = 128).  HBM-bound.
#include "common.cuh"
#include "internal.h"

namespace star {
namespace {

template <int D, bool OUT_BF16>
__global__ void __launch_bounds__(256) lse_merge_kernel(int parts_per_group, long long rows, const float* __restrict__ o_in,
                                                        const float* __restrict__ lse_in, void* __restrict__ o_out,
                                                        float* __restrict__ lse_out) {
  constexpr int PER = D / 32;
  const int lane = threadIdx.x % 32;
  const long long row = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int group = blockIdx.y;
  if (row >= rows) return;
  const long long part0 = (long long)group * parts_per_group;
  const int np = parts_per_group;

  // LSE statistics: the lanes take the partials 32 at a time.
  float m = -INFINITY;
  for (int i = lane; i < np; i += 32) {
    const float li = __ldg(lse_in + (part0 + i) * rows + row);
    if (isfinite(li)) m = fmaxf(m, li);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float lse = -INFINITY;
  if (m != -INFINITY) {
    float s = 0.f;
    for (int i = lane; i < np; i += 32) {
      const float li = __ldg(lse_in + (part0 + i) * rows + row);
      if (isfinite(li)) s += expf(li - m);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    lse = m + logf(s);
    // O: each lane owns PER consecutive columns; weights are broadcast from the lane
    // that computed them, and the loads of several partials are in flight at once.
    for (int base = 0; base < np; base += 32) {
      float w = 0.f;
      if (base + lane < np) {
        const float li = __ldg(lse_in + (part0 + base + lane) * rows + row);
        if (isfinite(li)) w = expf(li - lse);
      }
      const int cnt = min(32, np - base);
#pragma unroll 4
      for (int j = 0; j < cnt; ++j) {
        const float wj = __shfl_sync(0xffffffffu, w, j);
        const float* src = o_in + ((part0 + base + j) * rows + row) * D + lane * PER;
        if constexpr (PER == 4) {
          const float4 v = __ldg(reinterpret_cast<const float4*>(src));
          acc[0] = fmaf(wj, v.x, acc[0]);
          acc[1] = fmaf(wj, v.y, acc[1]);
          acc[2] = fmaf(wj, v.z, acc[2]);
          acc[3] = fmaf(wj, v.w, acc[3]);
        } else {
          const float2 v = __ldg(reinterpret_cast<const float2*>(src));
          acc[0] = fmaf(wj, v.x, acc[0]);
          acc[1] = fmaf(wj, v.y, acc[1]);
        }
      }
    }
  }
  const long long orow = (long long)group * rows + row;
  if (OUT_BF16) {
    bf16* dst = reinterpret_cast<bf16*>(o_out) + orow * D + lane * PER;
#pragma unroll
    for (int e = 0; e < PER; e += 2) *reinterpret_cast<uint32_t*>(dst + e) = pack_bf16x2(acc[e], acc[e + 1]);
  } else {
    float* dst = reinterpret_cast<float*>(o_out) + orow * D + lane * PER;
#pragma unroll
    for (int e = 0; e < PER; ++e) dst[e] = acc[e];
  }
  if (lane == 0 && lse_out) lse_out[orow] = lse;
}

}  // namespace

cudaError_t launch_lse_merge(int groups, int parts_per_group, int64_t rows, int d, const float* o_in,
                             const float* lse_in, void* o_out, bool out_bf16, float* lse_out, cudaStream_t st) {
  if (rows <= 0 || groups <= 0) return cudaSuccess;
  const int warps = 8;
  dim3 grid((unsigned)((rows + warps - 1) / warps), (unsigned)groups);
  if (d == 128) {
    if (out_bf16)
      lse_merge_kernel<128, true><<<grid, 32 * warps, 0, st>>>(parts_per_group, rows, o_in, lse_in, o_out, lse_out);
    else
      lse_merge_kernel<128, false><<<grid, 32 * warps, 0, st>>>(parts_per_group, rows, o_in, lse_in, o_out, lse_out);
  } else {
    if (out_bf16)
      lse_merge_kernel<64, true><<<grid, 32 * warps, 0, st>>>(parts_per_group, rows, o_in, lse_in, o_out, lse_out);
    else
      lse_merge_kernel<64, false><<<grid, 32 * warps, 0, st>>>(parts_per_group, rows, o_in, lse_in, o_out, lse_out);
  }
  return cudaGetLastError();
}

}  // namespace star
