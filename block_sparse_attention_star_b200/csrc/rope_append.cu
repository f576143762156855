// KV-cache writes of the Star Attention hot path (HBM-bound, no tensor cores).
//
// * rope_append: K rotated by RoPE at the token's position id and V copied,
//   both bf16, into the paged cache.  Phase 1 writes only the L context tokens
//   -- never the (n-1)*b anchor copies of c' ("Star Attention 完全拆解(一)",
//   "局部注意力与 KV 丢弃": the anchor's KV is discarded, and it equals block 1's
//   since the anchor keeps block 1's positions).  Phase 2 and decode append the
//   query / generated tokens at the tail of the last block ("仓库里的真实实现":
//   only the last host extends its cache).
// * zero_slots: clears cache slots past the context so that tiles which run over
//   the valid tail hold zeros, not stale values (masked keys get P = 0, and
//   0 * V must stay 0).
// * rope_q: the query heads rotated by RoPE once, before the attention kernel
//   (which then stages Q tiles by TMA instead of rotating them per work item).
// * rope_anchor: the anchor's keys roped at caller-given ids (anchor variants).
// * build_positions: the integer position ids of c' and the token -> (block,
//   page, slot) map ("被增广的上下文").
//
// Layout: pools are [num_pages][Hkv][P][d] bf16; logical page t / P of sequence
// bi is physical page page_table[bi * max_pages + t / P]; slot t % P.
// Each thread moves 16 bytes: for K, eight rotation pairs (x_j, x_{j+d/2}).
#include "common.cuh"
#include "internal.h"

#include <algorithm>

namespace star {
namespace {

struct RopeParams {
  double inv_freq[kMaxHalfDim];
};

// One thread per (sequence, token, 8-pair chunk): the 8 angles are computed once
// and applied to that chunk of every KV head of the token.
template <int D>
__global__ void __launch_bounds__(256) rope_append_kernel(const bf16* __restrict__ k, const bf16* __restrict__ v,
                                                          const int32_t* __restrict__ pos, int B, int ntok, int start,
                                                          int Hkv, bf16* __restrict__ kpool, bf16* __restrict__ vpool,
                                                          const int32_t* __restrict__ page_table, int max_pages,
                                                          int num_pages, int P, const __grid_constant__ RopeParams rp,
                                                          const __grid_constant__ SeqShift sh) {
  constexpr int CH = D / 16;
  const long long total = (long long)B * ntok * CH;
  for (long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x; gid < total;
       gid += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(gid % CH);
    const long long r = gid / CH;
    const int t = (int)(r % ntok);
    const int bi = (int)(r / ntok);
    const int slot_abs = start + (sh.on ? sh.delta[bi] : 0) + t;
    const int page = page_table[(size_t)bi * max_pages + slot_abs / P];
    if (page < 0 || page >= num_pages) {
      record_error(kDevBadPage);
      continue;
    }
    const int p_t = pos[(size_t)bi * ntok + t];
    double cs[4][2], sn[4][2];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      rope_sincos(p_t, rp.inv_freq[8 * c + 2 * e], cs[e][0], sn[e][0]);
      rope_sincos(p_t, rp.inv_freq[8 * c + 2 * e + 1], cs[e][1], sn[e][1]);
    }
    for (int h = 0; h < Hkv; ++h) {
      const size_t src = (((size_t)bi * ntok + t) * Hkv + h) * D;
      const size_t dst = (((size_t)page * Hkv + h) * P + (slot_abs % P)) * D;
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(k + src + 8 * c));
      const uint4 bq = __ldg(reinterpret_cast<const uint4*>(k + src + D / 2 + 8 * c));
      const uint32_t* aw = reinterpret_cast<const uint32_t*>(&a);
      const uint32_t* bw = reinterpret_cast<const uint32_t*>(&bq);
      uint32_t lo[4], hi[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) rope_rotate2(aw[e], bw[e], cs[e], sn[e], lo[e], hi[e]);
      *reinterpret_cast<uint4*>(kpool + dst + 8 * c) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      *reinterpret_cast<uint4*>(kpool + dst + D / 2 + 8 * c) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      // V: the same thread copies the two 16-byte chunks at the same offsets.
      *reinterpret_cast<uint4*>(vpool + dst + 8 * c) = __ldg(reinterpret_cast<const uint4*>(v + src + 8 * c));
      *reinterpret_cast<uint4*>(vpool + dst + D / 2 + 8 * c) =
          __ldg(reinterpret_cast<const uint4*>(v + src + D / 2 + 8 * c));
    }
  }
}

// RoPE of the query heads of ntok tokens per sequence: out[b][t][h] = rotation of
// q[b][t][h] at pos[b][t] (float64 rotation, one bf16 rounding, as the keys).  One
// thread per (head group, sequence, token, 8-pair chunk): the 8 angles are computed
// once and applied to that chunk of the group's hpt heads, four heads' loads in
// flight at a time.  Long inputs use one group of all H heads (each angle computed
// once); a few tokens split the heads over more threads, so that the kernel is not
// one serial chain of loads per thread.  out may be q itself: each element is read
// and then written by the same thread.
template <int D>
__global__ void __launch_bounds__(256) rope_q_kernel(const bf16* q, const int32_t* __restrict__ pos, int B, int ntok,
                                                     int H, int hpt, bf16* out, const __grid_constant__ RopeParams rp) {
  constexpr int CH = D / 16;
  const int HG = (H + hpt - 1) / hpt;
  const long long rows = (long long)B * ntok;
  const long long total = rows * CH * HG;
  for (long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x; gid < total;
       gid += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(gid % CH);
    const long long rest = gid / CH;
    const long long r = rest % rows;  // bi * ntok + t
    const int hg = (int)(rest / rows);
    const int p_t = pos[r];
    double cs[4][2], sn[4][2];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      rope_sincos(p_t, rp.inv_freq[8 * c + 2 * e], cs[e][0], sn[e][0]);
      rope_sincos(p_t, rp.inv_freq[8 * c + 2 * e + 1], cs[e][1], sn[e][1]);
    }
    const int h1 = min(H, (hg + 1) * hpt);
    for (int h0 = hg * hpt; h0 < h1; h0 += 4) {
      uint4 a[4], bq[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (h0 + u < h1) {
          const size_t off = ((size_t)r * H + h0 + u) * D;
          a[u] = *reinterpret_cast<const uint4*>(q + off + 8 * c);
          bq[u] = *reinterpret_cast<const uint4*>(q + off + D / 2 + 8 * c);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (h0 + u < h1) {
          const size_t off = ((size_t)r * H + h0 + u) * D;
          const uint32_t* aw = reinterpret_cast<const uint32_t*>(&a[u]);
          const uint32_t* bw = reinterpret_cast<const uint32_t*>(&bq[u]);
          uint32_t lo[4], hi[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) rope_rotate2(aw[e], bw[e], cs[e], sn[e], lo[e], hi[e]);
          *reinterpret_cast<uint4*>(out + off + 8 * c) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
          *reinterpret_cast<uint4*>(out + off + D / 2 + 8 * c) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        }
      }
    }
  }
}

// The anchor's keys roped at caller ids, one thread per (sequence, block, anchor token,
// 8-pair chunk): out[bi][i-1][h][j] = RoPE(k[bi][j][h], anchor_pos[bi][i-1][j]) for every KV head.
template <int D>
__global__ void __launch_bounds__(256) rope_anchor_kernel(const bf16* __restrict__ k, const int32_t* __restrict__ apos,
                                                          int B, int L, int nb, int a, int Hkv, bf16* __restrict__ out,
                                                          const __grid_constant__ RopeParams rp) {
  constexpr int CH = D / 16;
  const long long total = (long long)B * nb * a * CH;
  for (long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x; gid < total;
       gid += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(gid % CH);
    long long r = gid / CH;
    const int j = (int)(r % a);
    r /= a;  // bi * nb + block
    const int bi = (int)(r / nb);
    const int p_t = apos[r * a + j];
    double cs[4][2], sn[4][2];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      rope_sincos(p_t, rp.inv_freq[8 * c + 2 * e], cs[e][0], sn[e][0]);
      rope_sincos(p_t, rp.inv_freq[8 * c + 2 * e + 1], cs[e][1], sn[e][1]);
    }
    for (int h = 0; h < Hkv; ++h) {
      const size_t src = (((size_t)bi * L + j) * Hkv + h) * D;
      const size_t dst = ((size_t)(r * Hkv + h) * a + j) * D;
      const uint4 x = __ldg(reinterpret_cast<const uint4*>(k + src + 8 * c));
      const uint4 y = __ldg(reinterpret_cast<const uint4*>(k + src + D / 2 + 8 * c));
      const uint32_t* xw = reinterpret_cast<const uint32_t*>(&x);
      const uint32_t* yw = reinterpret_cast<const uint32_t*>(&y);
      uint32_t lo[4], hi[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) rope_rotate2(xw[e], yw[e], cs[e], sn[e], lo[e], hi[e]);
      *reinterpret_cast<uint4*>(out + dst + 8 * c) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      *reinterpret_cast<uint4*>(out + dst + D / 2 + 8 * c) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    }
  }
}

// Slots [from + delta[bi], to) of every sequence bi; `from` is the smallest start over the batch.
__global__ void zero_slots_kernel(int B, int from, int to, int Hkv, int d, bf16* kpool, bf16* vpool,
                                  const int32_t* page_table, int max_pages, int num_pages, int P,
                                  const __grid_constant__ SeqShift sh, int from_cap) {
  const int CH = d / 8;
  const long long span = to - from;
  const long long total = (long long)B * span * Hkv * CH;
  for (long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x; gid < total;
       gid += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(gid % CH);
    long long r = gid / CH;
    const int h = (int)(r % Hkv);
    r /= Hkv;
    const int s = from + (int)(r % span);
    const int bi = (int)(r / span);
    if (sh.on && s < from_cap + sh.delta[bi]) continue;  // still this sequence's context
    const int page = page_table[(size_t)bi * max_pages + s / P];
    if (page < 0 || page >= num_pages) {
      record_error(kDevBadPage);
      continue;
    }
    const size_t off = (((size_t)page * Hkv + h) * P + (s % P)) * d + 8 * c;
    *reinterpret_cast<uint4*>(kpool + off) = make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4*>(vpool + off) = make_uint4(0, 0, 0, 0);
  }
}

// Augmented row r of sequence bi: block 0 holds rows [0, b); block i >= 1 holds
// rows [b + (a+b)(i-1), b + (a+b) i): the a anchor rows (ids of tokens 0..a-1) then its own.
__global__ void build_positions_kernel(const int32_t* pos_ctx, int B, int L, int b, int anc,
                                       const int32_t* page_table, int max_pages, int P, int32_t* aug_pos,
                                       int32_t* block_map) {
  const int n = L / b;
  const long long aug_len = (long long)L + (long long)(n - 1) * anc;
  const long long total = (long long)B * aug_len;
  for (long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x; gid < total;
       gid += (long long)gridDim.x * blockDim.x) {
    const int bi = (int)(gid / aug_len);
    const long long r = gid % aug_len;
    long long tok;
    if (r < b) {
      tok = r;
    } else {
      const long long i = 1 + (r - b) / ((long long)anc + b);
      const long long off = (r - b) % ((long long)anc + b);
      tok = off < anc ? off : i * b + (off - anc);
    }
    aug_pos[gid] = pos_ctx[(size_t)bi * L + tok];
  }
  const long long total_map = (long long)B * L;
  for (long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x; gid < total_map;
       gid += (long long)gridDim.x * blockDim.x) {
    const int bi = (int)(gid / L);
    const int t = (int)(gid % L);
    block_map[3 * gid + 0] = t / b;
    block_map[3 * gid + 1] = page_table[(size_t)bi * max_pages + t / P];
    block_map[3 * gid + 2] = t % P;
  }
}

int grid_for(long long work, int threads) {
  long long g = (work + threads - 1) / threads;
  if (g < 1) g = 1;
  if (g > 148LL * 64) g = 148LL * 64;
  return (int)g;
}

}  // namespace

cudaError_t read_and_clear_error_rope(int* code) { return read_and_clear_tu_error(code); }

cudaError_t launch_rope_append(const void* k, const void* v, const int32_t* pos, int B, int ntok, int start, int Hkv,
                               int d, const CacheView& c, const RopeTable& rt, cudaStream_t st, const SeqShift* shift) {
  if (ntok <= 0 || B <= 0) return cudaSuccess;
  SeqShift sh;
  sh.on = 0;
  if (shift && shift->on) sh = *shift;
  RopeParams rp;
  for (int j = 0; j < d / 2; ++j) rp.inv_freq[j] = rt.inv_freq[j];
  const long long work = (long long)B * ntok * (d / 16);
  const int grid = grid_for(work, 256);
  if (d == 128) {
    rope_append_kernel<128><<<grid, 256, 0, st>>>(
        reinterpret_cast<const bf16*>(k), reinterpret_cast<const bf16*>(v), pos, B, ntok, start, Hkv,
        reinterpret_cast<bf16*>(c.k_pool), reinterpret_cast<bf16*>(c.v_pool), c.page_table, c.max_pages,
        c.num_pages, c.P, rp, sh);
  } else {
    rope_append_kernel<64><<<grid, 256, 0, st>>>(
        reinterpret_cast<const bf16*>(k), reinterpret_cast<const bf16*>(v), pos, B, ntok, start, Hkv,
        reinterpret_cast<bf16*>(c.k_pool), reinterpret_cast<bf16*>(c.v_pool), c.page_table, c.max_pages,
        c.num_pages, c.P, rp, sh);
  }
  return cudaGetLastError();
}

cudaError_t launch_rope_q(const void* q, const int32_t* pos, int B, int ntok, int H, int d, void* out,
                          const RopeTable& rt, cudaStream_t st) {
  if (ntok <= 0 || B <= 0) return cudaSuccess;
  RopeParams rp;
  for (int j = 0; j < d / 2; ++j) rp.inv_freq[j] = rt.inv_freq[j];
  // Head groups: enough threads to fill the GPU (148 SMs x 1024), at most one head each.
  const long long base = (long long)B * ntok * (d / 16);
  const long long groups = std::min<long long>(H, std::max<long long>(1, 148LL * 1024 / base));
  const int hpt = (int)((H + groups - 1) / groups);
  const int grid = grid_for(base * ((H + hpt - 1) / hpt), 256);
  if (d == 128)
    rope_q_kernel<128><<<grid, 256, 0, st>>>(reinterpret_cast<const bf16*>(q), pos, B, ntok, H, hpt,
                                             reinterpret_cast<bf16*>(out), rp);
  else
    rope_q_kernel<64><<<grid, 256, 0, st>>>(reinterpret_cast<const bf16*>(q), pos, B, ntok, H, hpt,
                                            reinterpret_cast<bf16*>(out), rp);
  return cudaGetLastError();
}

cudaError_t launch_zero_slots(int B, int from, int to, int Hkv, int d, const CacheView& c, cudaStream_t st,
                              const SeqShift* shift) {
  SeqShift sh;
  sh.on = 0;
  int lo = from;
  if (shift && shift->on) {
    sh = *shift;
    for (int i = 0; i < B; ++i) lo = std::min(lo, from + sh.delta[i]);
  }
  if (to <= lo) return cudaSuccess;
  const long long work = (long long)B * (to - lo) * Hkv * (d / 8);
  zero_slots_kernel<<<grid_for(work, 256), 256, 0, st>>>(B, lo, to, Hkv, d, reinterpret_cast<bf16*>(c.k_pool),
                                                          reinterpret_cast<bf16*>(c.v_pool), c.page_table,
                                                          c.max_pages, c.num_pages, c.P, sh, from);
  return cudaGetLastError();
}

cudaError_t launch_build_positions(const int32_t* pos_ctx, int B, int L, int b, int a, const CacheView& c,
                                   int32_t* aug_pos, int32_t* block_map, cudaStream_t st) {
  const long long work = (long long)B * (L + (long long)(L / b - 1) * a);
  build_positions_kernel<<<grid_for(work, 256), 256, 0, st>>>(pos_ctx, B, L, b, a, c.page_table, c.max_pages, c.P,
                                                               aug_pos, block_map);
  return cudaGetLastError();
}

cudaError_t launch_rope_anchor(const void* k, const int32_t* anchor_pos, int B, int L, int n, int a, int Hkv, int d,
                               void* out, const RopeTable& rt, cudaStream_t st) {
  if (n <= 1 || a <= 0) return cudaSuccess;
  RopeParams rp;
  for (int j = 0; j < d / 2; ++j) rp.inv_freq[j] = rt.inv_freq[j];
  const long long work = (long long)B * (n - 1) * a * (d / 16);
  const int grid = grid_for(work, 256);
  if (d == 128)
    rope_anchor_kernel<128><<<grid, 256, 0, st>>>(reinterpret_cast<const bf16*>(k), anchor_pos, B, L, n - 1, a, Hkv,
                                                  reinterpret_cast<bf16*>(out), rp);
  else
    rope_anchor_kernel<64><<<grid, 256, 0, st>>>(reinterpret_cast<const bf16*>(k), anchor_pos, B, L, n - 1, a, Hkv,
                                                 reinterpret_cast<bf16*>(out), rp);
  return cudaGetLastError();
}

}  // namespace star
