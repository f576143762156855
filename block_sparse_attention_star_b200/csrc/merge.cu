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

  float m = -INFINITY;
  for (int i = 0; i < parts_per_group; ++i) {
    const float li = lse_in[(part0 + i) * rows + row];
    if (isfinite(li)) m = fmaxf(m, li);
  }
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float lse = -INFINITY;
  if (m != -INFINITY) {
    float s = 0.f;
    for (int i = 0; i < parts_per_group; ++i) {
      const float li = lse_in[(part0 + i) * rows + row];
      if (isfinite(li)) s += expf(li - m);
    }
    lse = m + logf(s);
    for (int i = 0; i < parts_per_group; ++i) {
      const float li = lse_in[(part0 + i) * rows + row];
      if (!isfinite(li)) continue;
      const float w = expf(li - lse);
      const float* src = o_in + ((part0 + i) * rows + row) * D + lane * PER;
      if constexpr (PER == 4) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(src));
        acc[0] += w * v.x;
        acc[1] += w * v.y;
        acc[2] += w * v.z;
        acc[3] += w * v.w;
      } else {
        const float2 v = __ldg(reinterpret_cast<const float2*>(src));
        acc[0] += w * v.x;
        acc[1] += w * v.y;
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
