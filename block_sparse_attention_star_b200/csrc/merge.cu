// Exact merge of attention partials (O_i, LSE_i) into global attention
// ("Star Attention 完全拆解(一)", "组装全局结果": s_global = sum_h s_h and
// A_global = sum_h (s_h / s_global) A_h; "数值稳定性": carried out on
// log-sum-exp values in float32, then cast to the query dtype).
//
// With m = max_i LSE_i over the partials whose LSE is finite,
//   LSE = m + log(sum_i exp(LSE_i - m)),   O = sum_i exp(LSE_i - LSE) O_i.
// A partial with a non-finite LSE (an empty block: -inf) contributes nothing,
// and its O is never read into the sum (an empty partial's O may be 0/0); a row
// with no finite partial gives O = 0, LSE = -inf.  A NaN or +inf LSE cannot come
// from a correct partial: it is skipped the same way and also recorded in the
// device error word (kDevBadPartial), which star_device_status reports.
//
// One warp per output row; each lane owns d/32 consecutive columns (one
// 16-byte load per partial at d = 128).  The kernel keeps memory round trips few:
// the first batch of O loads is issued before the LSE statistics are read, the
// statistics are one online (max, sum) pass, and the O partials stream in batches
// of kBatch loads.  Decode-sized merges (few rows, 17..64 partials) take a variant
// with two warps per row that loads every partial in one batch.
#include "common.cuh"
#include "internal.h"

namespace star {
namespace {

constexpr int kBatch = 16;

template <int D>
struct Cols;
template <>
struct Cols<128> {
  using T = float4;
  static __device__ __forceinline__ void fma(float* acc, float w, const T& v) {
    acc[0] = fmaf(w, v.x, acc[0]);
    acc[1] = fmaf(w, v.y, acc[1]);
    acc[2] = fmaf(w, v.z, acc[2]);
    acc[3] = fmaf(w, v.w, acc[3]);
  }
};
template <>
struct Cols<64> {
  using T = float2;
  static __device__ __forceinline__ void fma(float* acc, float w, const T& v) {
    acc[0] = fmaf(w, v.x, acc[0]);
    acc[1] = fmaf(w, v.y, acc[1]);
  }
};

template <int D, bool OUT_BF16>
__global__ void __launch_bounds__(256) lse_merge_kernel(int parts_per_group, long long rows, const float* __restrict__ o_in,
                                                        const float* __restrict__ lse_in, void* __restrict__ o_out,
                                                        float* __restrict__ lse_out) {
  constexpr int PER = D / 32;
  using V = typename Cols<D>::T;
  griddep_wait();  // the partials come from the previous kernel
  griddep_launch_dependents();
  const int lane = threadIdx.x % 32;
  const long long row = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int group = blockIdx.y;
  if (row >= rows) return;
  const long long part0 = (long long)group * parts_per_group;
  const int np = parts_per_group;
  const float* ob = o_in + (part0 * rows + row) * D + lane * PER;  // partial i at ob + i * rows * D
  const float* lb = lse_in + part0 * rows + row;                   // partial i at lb + i * rows
  const size_t ostride = (size_t)rows * D;

  V v[kBatch];
#pragma unroll
  for (int j = 0; j < kBatch; ++j)
    if (j < np) v[j] = __ldg(reinterpret_cast<const V*>(ob + j * ostride));

  // LSE statistics: online (max, sum) over the lane's partials, then across lanes.
  float m = -INFINITY, s = 0.f;
  bool bad = false;
  for (int i = lane; i < np; i += 32) {
    const float li = __ldg(lb + (size_t)i * rows);
    if (!isfinite(li)) {
      bad |= !(li == -INFINITY);
      continue;
    }
    if (li > m) {
      s = s * expf(m - li) + 1.f;
      m = li;
    } else {
      s += expf(li - m);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float mo = __shfl_xor_sync(0xffffffffu, m, off), so = __shfl_xor_sync(0xffffffffu, s, off);
    const float mm = fmaxf(m, mo);
    if (mm != -INFINITY) s = (m == -INFINITY ? 0.f : s * expf(m - mm)) + (mo == -INFINITY ? 0.f : so * expf(mo - mm));
    m = mm;
  }
  const float lse = (m == -INFINITY) ? -INFINITY : m + logf(s);
  if (bad) record_error(kDevBadPartial);

  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  if (m != -INFINITY) {
    for (int base = 0; base < np; base += kBatch) {
      if (base > 0) {
#pragma unroll
        for (int j = 0; j < kBatch; ++j)
          if (base + j < np) v[j] = __ldg(reinterpret_cast<const V*>(ob + (size_t)(base + j) * ostride));
      }
      // Lane j holds the weight of partial base + j; a non-finite LSE weighs 0.
      float w = 0.f;
      if (lane < kBatch && base + lane < np) {
        const float li = __ldg(lb + (size_t)(base + lane) * rows);
        if (isfinite(li)) w = expf(li - lse);
      }
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const float wj = __shfl_sync(0xffffffffu, w, j);
        if (base + j < np && wj != 0.f) Cols<D>::fma(acc, wj, v[j]);
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

// Decode-sized merges (a few dozen rows, 17..64 partials): two warps per row, each loading
// its half of the partials (at most 32: O and LSE) in one batch, so the merge is a single
// memory round trip; the halves' statistics and sums meet in shared memory.  Four rows per
// block of 8 warps; every thread reaches both barriers (no early exit).
template <int D, bool OUT_BF16>
__global__ void __launch_bounds__(256) lse_merge_pair_kernel(int parts_per_group, long long rows,
                                                             const float* __restrict__ o_in,
                                                             const float* __restrict__ lse_in,
                                                             void* __restrict__ o_out, float* __restrict__ lse_out) {
  constexpr int PER = D / 32;
  using V = typename Cols<D>::T;
  __shared__ float st[4][2][2];        // [row slot][half]: (max, sum)
  __shared__ float acc_sh[4][D];       // [row slot]: half 1's weighted sum
  griddep_wait();  // the partials come from the previous kernel
  griddep_launch_dependents();
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  const int slot = warp >> 1, half = warp & 1;
  const long long row = (long long)blockIdx.x * 4 + slot;
  const int group = blockIdx.y;
  const bool live = row < rows;
  const int np = parts_per_group;
  const int h0 = half ? (np + 1) / 2 : 0;
  const int nh = (half ? np : (np + 1) / 2) - h0;  // <= 32
  const long long part0 = (long long)group * np + h0;
  const float* ob = o_in + (part0 * rows + row) * D + lane * PER;
  const size_t ostride = (size_t)rows * D;
  V v[32];
#pragma unroll
  for (int j = 0; j < 32; ++j)
    if (live && j < nh) v[j] = __ldg(reinterpret_cast<const V*>(ob + j * ostride));
  const float li = (live && lane < nh) ? __ldg(lse_in + (part0 + lane) * rows + row) : -INFINITY;
  const bool fin = isfinite(li);
  if (!fin && !(li == -INFINITY)) record_error(kDevBadPartial);
  float m = fin ? li : -INFINITY;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float sum = (fin && m != -INFINITY) ? expf(li - m) : 0.f;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if (lane == 0) {
    st[slot][half][0] = m;
    st[slot][half][1] = sum;
  }
  __syncthreads();
  const float mo = st[slot][half ^ 1][0], so = st[slot][half ^ 1][1];
  const float mm = fmaxf(m, mo);
  float lse = -INFINITY;
  if (mm != -INFINITY)
    lse = mm + logf((m == -INFINITY ? 0.f : sum * expf(m - mm)) + (mo == -INFINITY ? 0.f : so * expf(mo - mm)));
  const float w = (fin && lse != -INFINITY) ? expf(li - lse) : 0.f;  // this lane's partial's weight
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float wj = __shfl_sync(0xffffffffu, w, j);
    if (j < nh && wj != 0.f) Cols<D>::fma(acc, wj, v[j]);
  }
  if (half == 1) {
#pragma unroll
    for (int e = 0; e < PER; ++e) acc_sh[slot][lane * PER + e] = acc[e];
  }
  __syncthreads();
  if (half == 0 && live) {
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] += acc_sh[slot][lane * PER + e];
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
}

}  // namespace

cudaError_t read_and_clear_error_merge(int* code) { return read_and_clear_tu_error(code); }

cudaError_t launch_lse_merge(int groups, int parts_per_group, int64_t rows, int d, const float* o_in,
                             const float* lse_in, void* o_out, bool out_bf16, float* lse_out, cudaStream_t st) {
  if (rows <= 0 || groups <= 0) return cudaSuccess;
  const long long nrows0 = rows;
  if (parts_per_group > kBatch && parts_per_group <= 64 && rows <= 4096) {
    const dim3 grid((unsigned)((rows + 3) / 4), (unsigned)groups);
    auto kern = d == 128 ? (out_bf16 ? lse_merge_pair_kernel<128, true> : lse_merge_pair_kernel<128, false>)
                         : (out_bf16 ? lse_merge_pair_kernel<64, true> : lse_merge_pair_kernel<64, false>);
    return launch_pdl(kern, grid, 256, 0, st, parts_per_group, nrows0, o_in, lse_in, o_out, lse_out);
  }
  const int warps = 8;
  const dim3 grid((unsigned)((rows + warps - 1) / warps), (unsigned)groups);
  const long long nrows = rows;
  auto kern = d == 128 ? (out_bf16 ? lse_merge_kernel<128, true> : lse_merge_kernel<128, false>)
                       : (out_bf16 ? lse_merge_kernel<64, true> : lse_merge_kernel<64, false>);
  return launch_pdl(kern, grid, 32 * warps, 0, st, parts_per_group, nrows, o_in, lse_in, o_out, lse_out);
}

}  // namespace star
