// The Phase-2 star exchange over peer memory: every GPU owns a block range and
// contributes, per query call and per decode token, one (output, log-sum-exp)
// partial per block ("Star Attention 完全拆解(一)", "通信量:每层每 token 一个标量加
// 一个向量"; merged exactly as in "组装全局结果").  The pages gather them with a
// blocking all_gather of out, one of lse, then a barrier.  Here:
//
//  * merge_scatter_kernel merges a rank's chunk partials into its per-block partials
//    (the chunks exist only to fill the GPU) and stores every result row straight into
//    slot `rank` of EVERY rank's exchange buffer (plain stores to peer memory over
//    NVLink; nothing is staged).  The last block to finish publishes ready = epoch in
//    each buffer with a system-scope release.
//  * gather_merge_kernel waits (bounded) until all ranks' ready words of its own buffer
//    show the epoch, merges the world x slots partials it holds, and its last block
//    tells every rank, through that rank's ack word, that the slots may be reused.
//  * A rank writes into parity (epoch & 1) and first waits until every rank has acked
//    epoch - 2 (the last use of that parity), so the exchange needs no barrier.
//
// Layout of one rank's buffer (star_exchange_size): a 256-byte header
//   u64 ready[2][8]   ready[p][w]: epoch whose parity-p data from rank w is in place
//   u64 ack[8]        ack[w]: last epoch rank w finished merging (from its own buffer)
//   u32 scatter_done, gather_done  (block counters of this rank's own kernels)
// then [2 parities][world slots] of { f32 O [slots][rows][d]; f32 LSE [slots][rows] }.
#include "star.h"
#include "common.cuh"
#include "internal.h"

#include <cstring>

namespace star {
namespace {

constexpr int kMaxWorld = 8;
constexpr size_t kHeader = 256;

struct Header {
  unsigned long long ready[2][kMaxWorld];
  unsigned long long ack[kMaxWorld];
  unsigned int scatter_done, gather_done;
};
static_assert(sizeof(Header) <= kHeader, "exchange header");

__host__ __device__ inline size_t rup(size_t x, size_t m) { return (x + m - 1) / m * m; }

struct XLayout {
  size_t o_bytes, slot_bytes;  // one rank's slot: O [slots][rows][d] then LSE [slots][rows]
};
__host__ __device__ inline XLayout xlayout(int slots, long long rows, int d) {
  XLayout l;
  l.o_bytes = rup((size_t)slots * rows * d * 4, 256);
  l.slot_bytes = l.o_bytes + rup((size_t)slots * rows * 4, 256);
  return l;
}

struct XParams {
  unsigned char* peers[kMaxWorld];  // every rank's buffer as mapped here (peers[rank] = own)
  int world, rank;
  int slots;                        // partials per rank per exchange
  long long rows;
  unsigned long long epoch;
};

__device__ __forceinline__ unsigned long long ld_acquire_sys(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.sys.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_sys(unsigned long long* p, unsigned long long v) {
  asm volatile("st.release.sys.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Thread 0 of the block waits until words[w] (w < world) satisfy pred; bounded by the
// translation unit's wait limit, after which kDevTimeoutExchange is recorded and the
// block goes on (its results are then not to be trusted: star_device_status says so).
template <typename Pred>
__device__ __forceinline__ bool wait_words(const unsigned long long* words, int world, Pred pred) {
  __shared__ int ok_sh;
  if (threadIdx.x == 0) {
    int ok = 1;
    const uint64_t t0 = globaltimer_ns();
    for (int w = 0; w < world && ok; ++w) {
      while (!pred(ld_acquire_sys(words + w))) {
        if (globaltimer_ns() - t0 > g_wait_limit_ns) {
          record_error(kDevTimeoutExchange);
          ok = 0;
          break;
        }
        __nanosleep(256);
      }
    }
    ok_sh = ok;
  }
  __syncthreads();
  return ok_sh != 0;
}

template <int D>
struct XCols;
template <>
struct XCols<128> {
  using T = float4;
};
template <>
struct XCols<64> {
  using T = float2;
};

__device__ __forceinline__ void vfma(float* acc, float w, const float4& v) {
  acc[0] = fmaf(w, v.x, acc[0]);
  acc[1] = fmaf(w, v.y, acc[1]);
  acc[2] = fmaf(w, v.z, acc[2]);
  acc[3] = fmaf(w, v.w, acc[3]);
}
__device__ __forceinline__ void vfma(float* acc, float w, const float2& v) {
  acc[0] = fmaf(w, v.x, acc[0]);
  acc[1] = fmaf(w, v.y, acc[1]);
}

// Merge of np partials of one row (lane owns d/32 columns): partial i's O at o(i), LSE at
// l(i).  A non-finite LSE contributes nothing (an empty block's -inf; NaN / +inf are also
// recorded).  Returns the row's LSE; acc holds the merged O.
template <int D, bool FROM_PEERS, typename OPtr, typename LPtr>
__device__ __forceinline__ float merge_row(int np, OPtr o, LPtr l, int lane, float (&acc)[D / 32]) {
  using V = typename XCols<D>::T;
  float m = -INFINITY, s = 0.f;
  bool bad = false;
  for (int i = lane; i < np; i += 32) {
    const float li = l(i);
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
  if (bad) record_error(kDevBadPartial);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float mo = __shfl_xor_sync(0xffffffffu, m, off), so = __shfl_xor_sync(0xffffffffu, s, off);
    const float mm = fmaxf(m, mo);
    if (mm != -INFINITY) s = (m == -INFINITY ? 0.f : s * expf(m - mm)) + (mo == -INFINITY ? 0.f : so * expf(mo - mm));
    m = mm;
  }
  const float lse = (m == -INFINITY) ? -INFINITY : m + logf(s);
#pragma unroll
  for (int e = 0; e < D / 32; ++e) acc[e] = 0.f;
  if (m != -INFINITY) {
    for (int i = 0; i < np; ++i) {
      const float li = l(i);
      if (!isfinite(li)) continue;
      const V* src = reinterpret_cast<const V*>(o(i) + lane * (D / 32));
      vfma(acc, expf(li - lse), FROM_PEERS ? __ldcg(src) : __ldg(src));  // peers' rows: read from L2
    }
  }
  return lse;
}

// One warp per (slot, row): slot g < n_groups merges its group's parts_per_group chunk
// partials (o_in [n_groups * ppg][rows][d], lse_in [..][rows]); slots [n_groups, slots)
// are empty partials.  Every result row goes to slot `rank` of every rank's buffer.
template <int D>
__global__ void __launch_bounds__(256) merge_scatter_kernel(const __grid_constant__ XParams xp, int n_groups, int ppg,
                                                            const float* __restrict__ o_in,
                                                            const float* __restrict__ lse_in) {
  griddep_wait();  // the chunk partials come from the previous kernel
  const XLayout lay = xlayout(xp.slots, xp.rows, D);
  const int par = (int)(xp.epoch & 1ull);
  Header* own = reinterpret_cast<Header*>(xp.peers[xp.rank]);
  // The parity's slots in every rank's buffer are free once every rank acked epoch - 2.
  const unsigned long long need = xp.epoch >= 2 ? xp.epoch - 2 : 0;
  wait_words(own->ack, xp.world, [need](unsigned long long v) { return v >= need; });
  const int lane = threadIdx.x % 32;
  const long long gw = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;  // global warp
  const long long total = (long long)xp.slots * xp.rows;
  if (gw < total) {
    const int g = (int)(gw / xp.rows);
    const long long row = gw - (long long)g * xp.rows;
    float acc[D / 32];
    float lse = -INFINITY;
    if (g < n_groups) {
      const size_t ostride = (size_t)xp.rows * D;
      const float* ob = o_in + ((size_t)g * ppg * xp.rows + row) * D;
      const float* lb = lse_in + (size_t)g * ppg * xp.rows + row;
      lse = merge_row<D, false>(
          ppg, [&](int i) { return ob + (size_t)i * ostride; }, [&](int i) { return __ldg(lb + (size_t)i * xp.rows); },
          lane, acc);
    } else {
#pragma unroll
      for (int e = 0; e < D / 32; ++e) acc[e] = 0.f;
    }
    const size_t orow = ((size_t)g * xp.rows + row) * D + lane * (D / 32);
    const size_t lrow = (size_t)g * xp.rows + row;
    for (int w = 0; w < xp.world; ++w) {
      unsigned char* slot = xp.peers[w] + kHeader + ((size_t)par * xp.world + xp.rank) * lay.slot_bytes;
      float* dst = reinterpret_cast<float*>(slot) + orow;
#pragma unroll
      for (int e = 0; e < D / 32; ++e) dst[e] = acc[e];
      if (lane == 0) reinterpret_cast<float*>(slot + lay.o_bytes)[lrow] = lse;
    }
  }
  // The last block to finish publishes the epoch in every buffer (release: the rows
  // stored by every block happen before it).
  __threadfence_system();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned int prev = atomicAdd(&own->scatter_done, 1u);
    if (prev == gridDim.x - 1) {
      own->scatter_done = 0;
      __threadfence_system();
      for (int w = 0; w < xp.world; ++w) {
        Header* h = reinterpret_cast<Header*>(xp.peers[w]);
        st_release_sys(&h->ready[par][xp.rank], xp.epoch);
      }
    }
  }
  griddep_launch_dependents();
}

// One warp per row: waits for every rank's slot of this epoch, merges the world x slots
// partials of the row (bf16 out, f32 LSE), then the last block acks the epoch to every rank.
template <int D>
__global__ void __launch_bounds__(256) gather_merge_kernel(const __grid_constant__ XParams xp, bf16* __restrict__ out,
                                                           float* __restrict__ lse_out) {
  griddep_wait();
  const XLayout lay = xlayout(xp.slots, xp.rows, D);
  const int par = (int)(xp.epoch & 1ull);
  unsigned char* base = xp.peers[xp.rank];
  Header* own = reinterpret_cast<Header*>(base);
  const unsigned long long ep = xp.epoch;
  wait_words(own->ready[par], xp.world, [ep](unsigned long long v) { return v == ep; });
  const int lane = threadIdx.x % 32;
  const long long row = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (row < xp.rows) {
    const unsigned char* par0 = base + kHeader + (size_t)par * xp.world * lay.slot_bytes;
    const int np = xp.world * xp.slots;
    auto o = [&](int i) {
      const int w = i / xp.slots, k = i - (i / xp.slots) * xp.slots;
      return reinterpret_cast<const float*>(par0 + (size_t)w * lay.slot_bytes) + ((size_t)k * xp.rows + row) * D;
    };
    auto l = [&](int i) {
      const int w = i / xp.slots, k = i - (i / xp.slots) * xp.slots;
      return __ldcg(reinterpret_cast<const float*>(par0 + (size_t)w * lay.slot_bytes + lay.o_bytes) +
                    (size_t)k * xp.rows + row);
    };
    float acc[D / 32];
    const float lse = merge_row<D, true>(np, o, l, lane, acc);
    bf16* dst = out + row * D + lane * (D / 32);
#pragma unroll
    for (int e = 0; e < D / 32; e += 2) *reinterpret_cast<uint32_t*>(dst + e) = pack_bf16x2(acc[e], acc[e + 1]);
    if (lane == 0 && lse_out) lse_out[row] = lse;
  }
  // Every block has read its rows: the last one acks the epoch to every rank.
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned int prev = atomicAdd(&own->gather_done, 1u);
    if (prev == gridDim.x - 1) {
      own->gather_done = 0;
      __threadfence_system();
      for (int w = 0; w < xp.world; ++w) {
        Header* h = reinterpret_cast<Header*>(xp.peers[w]);
        st_release_sys(&h->ack[xp.rank], ep);
      }
    }
  }
  griddep_launch_dependents();
}

}  // namespace

size_t exchange_bytes(int world, int slots, long long rows, int d) {
  return kHeader + (size_t)2 * world * xlayout(slots, rows, d).slot_bytes;
}

cudaError_t launch_merge_scatter(const ExchangeView& x, int n_groups, int ppg, long long rows, int d, const float* o_in,
                                 const float* lse_in, unsigned long long epoch, cudaStream_t st) {
  XParams p;
  memset(&p, 0, sizeof(p));
  for (int w = 0; w < x.world; ++w) p.peers[w] = reinterpret_cast<unsigned char*>(x.peers[w]);
  p.world = x.world;
  p.rank = x.rank;
  p.slots = x.slots;
  p.rows = rows;
  p.epoch = epoch;
  const long long warps = (long long)x.slots * rows;
  const dim3 grid((unsigned)((warps + 7) / 8));
  auto kern = d == 128 ? merge_scatter_kernel<128> : merge_scatter_kernel<64>;
  return launch_pdl(kern, grid, 256, 0, st, p, n_groups, ppg, o_in, lse_in);
}

cudaError_t launch_gather_merge(const ExchangeView& x, long long rows, int d, unsigned long long epoch, void* out,
                                float* lse_out, cudaStream_t st) {
  XParams p;
  memset(&p, 0, sizeof(p));
  for (int w = 0; w < x.world; ++w) p.peers[w] = reinterpret_cast<unsigned char*>(x.peers[w]);
  p.world = x.world;
  p.rank = x.rank;
  p.slots = x.slots;
  p.rows = rows;
  p.epoch = epoch;
  const dim3 grid((unsigned)((rows + 7) / 8));
  auto kern = d == 128 ? gather_merge_kernel<128> : gather_merge_kernel<64>;
  return launch_pdl(kern, grid, 256, 0, st, p, reinterpret_cast<bf16*>(out), lse_out);
}

cudaError_t read_and_clear_error_exchange(int* code) { return read_and_clear_tu_error(code); }
cudaError_t set_debug_exchange(unsigned long long wait_limit_ns, int flags) {
  return set_tu_debug(wait_limit_ns, flags);
}

}  // namespace star
