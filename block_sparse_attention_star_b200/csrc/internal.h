// Internal launch interfaces between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>
#include <utility>

namespace star {

// A kernel that uses more than 48 KB of dynamic shared memory must opt in once per
// device.  `done` (one per kernel) remembers the devices (ordinals < 64) already set,
// so a process that drives several GPUs opts in on each of them.
inline cudaError_t opt_in_dynamic_smem(const void* kern, int bytes, std::atomic<unsigned long long>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_release);
  return e;
}

// SM count of the current device (looked up once per device; 148 if the query fails).
int current_device_sm_count();

// A launch with programmatic stream serialization: the kernel may start while the
// previous kernel in the stream drains, and waits (griddepcontrol.wait) before it
// touches global memory.
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

constexpr int kMaxHalfDimHost = 64;
constexpr int kMaxVarB = 256;   // sequences of a batch with per-sequence lengths (passed by value)

// Per-sequence shift of cache indices: a batch with per-sequence context lengths
// L_s keeps sequence s's tail at L_s, i.e. index x of the capacity frame maps to
// x + delta[s] with delta[s] = L_s - L.  on = 0: every sequence has L tokens.
struct SeqShift {
  int on;
  int delta[kMaxVarB];
};

struct RopeTable {
  double inv_freq[kMaxHalfDimHost];   // theta^(-2j/d), j < d/2
};

// Paged KV cache view (see star.h: pools are [num_pages][Hkv][P][d] bf16).
struct CacheView {
  void* k_pool;
  void* v_pool;
  const int32_t* page_table;
  int max_pages;
  int num_pages;
  int P;
};

// --- rope_append.cu -------------------------------------------------------
// RoPE(K) at `pos` and copy of V for ntok tokens per sequence, written at cache
// slots [start, start + ntok).  k/v: [B][ntok][Hkv][d] bf16, pos: [B][ntok].
// shift (may be NULL): sequence s writes slots [start + delta[s], ...).
cudaError_t launch_rope_append(const void* k, const void* v, const int32_t* pos, int B, int ntok, int start,
                               int Hkv, int d, const CacheView& c, const RopeTable& rt, cudaStream_t st,
                               const SeqShift* shift = nullptr);
// RoPE of all H query heads of ntok tokens: out = rotate(q) at pos (out may be q).
// q/out: [B][ntok][H][d] bf16, pos: [B][ntok].
cudaError_t launch_rope_q(const void* q, const int32_t* pos, int B, int ntok, int H, int d, void* out,
                          const RopeTable& rt, cudaStream_t st);
// Zero cache slots [from, to) of every sequence (K and V).
// shift (may be NULL): sequence s clears slots [from + delta[s], to).
cudaError_t launch_zero_slots(int B, int from, int to, int Hkv, int d, const CacheView& c, cudaStream_t st,
                              const SeqShift* shift = nullptr);
// c' position ids [B][L + (n-1) a] (anchor = the first a tokens) and block map [B][L][3].
cudaError_t launch_build_positions(const int32_t* pos_ctx, int B, int L, int b, int a, const CacheView& c,
                                   int32_t* aug_pos, int32_t* block_map, cudaStream_t st);
// The anchor's keys roped at caller ids: out[bi][i-1][h][j] = RoPE(k[bi][j][h], anchor_pos[bi][i-1][j])
// for blocks i = 1..n-1 (0-based), j < a.  k: [B][L][Hkv][d] bf16; out: bf16 [B][n-1][Hkv][a][d].
cudaError_t launch_rope_anchor(const void* k, const int32_t* anchor_pos, int B, int L, int n, int a, int Hkv, int d,
                               void* out, const RopeTable& rt, cudaStream_t st);

// --- merge.cu ---------------------------------------------------------------
// groups x rows outputs; group g merges input parts [g*parts_per_group, (g+1)*parts_per_group).
// o_in: [parts][rows][d] f32, lse_in: [parts][rows].  Output bf16 or f32 [groups][rows][d].
cudaError_t launch_lse_merge(int groups, int parts_per_group, int64_t rows, int d, const float* o_in,
                             const float* lse_in, void* o_out, bool out_bf16, float* lse_out, cudaStream_t st);

// --- attn_sm100.cu ------------------------------------------------------------
struct AttnLaunch {
  int mode;               // 0: Phase-1 context attention, 1: Phase-2 query partials
  int B, Hq, Hkv, d, L, b, n;
  const void* q;          // [B][Ntok][Hq][d] bf16, already rotated (mode 0: staged by TMA, mode 1: by threads)
  int Ntok;
  CacheView cache;
  void* out_bf16;         // mode 0: [B][L][Hq][d]
  float* out_f32;         // mode 1: [parts][B][T][Hq][d]
  float* lse_f32;         // mode 1: [parts][B][T][Hq]
  int chunks_per_block;   // mode 1
  int anchor;             // mode 0: anchor size a (the first a keys of block 1)
  SeqShift shift;         // per-sequence context lengths L + delta[s] (on = 0: all L)
  const void* anchor_k;   // mode 0: NULL (anchor keys are block 1's cached keys) or bf16 [B][n-1][Hkv][a][d]
  float scale_log2;
  // A shard: blocks [blk0, blk0 + nblk) of every sequence (nblk = 0: through the last block).
  // Mode 0: q and out hold the range's nblk * b rows per sequence.  Mode 1: parts are the
  // range's chunks; the query tail is the last block's unless no_tail.
  int blk0, nblk, no_tail;
};
int attn_num_parts(const AttnLaunch& a);  // mode 1: n * chunks_per_block
cudaError_t launch_attention(const AttnLaunch& a, cudaStream_t st, const char** why);

// --- decode.cu ----------------------------------------------------------------
struct DecodeLaunch {
  int B, Hq, Hkv, d;
  const void* q;          // [B][Hq][d] bf16 (pre-RoPE)
  const void* k_new;      // [B][Hkv][d] bf16 (pre-RoPE): appended at slot n_keys - 1 by the kernel
  const void* v_new;      // [B][Hkv][d] bf16
  const int32_t* pos;     // [B] position of the decoded token
  int n_keys;             // keys [k_lo, n_keys) of every sequence (the longest, with a shift)
  int k_lo;               // first key: 0, or a shard's first key (a multiple of 128; no shift then)
  int append;             // 1: slot n_keys - 1 is the new token's, appended by the kernel
  SeqShift shift;         // sequence s has n_keys + delta[s] keys
  int chunk;              // keys per CTA
  CacheView cache;
  float* o_ws;            // [nchunks][B*Hq][d]
  float* lse_ws;          // [nchunks][B*Hq]
  float scale_log2;
  RopeTable rope;
};
int decode_num_chunks(int n_keys, int chunk);
int decode_pick_chunk(int B, int Hkv, int G, int n_keys, int num_sms);
int decode_pick_chunk_var(int B, int Hkv, const int* n_keys_of, int min_chunk, int num_sms);
cudaError_t launch_decode(const DecodeLaunch& a, cudaStream_t st);

// --- exchange.cu: the Phase-2 star exchange over peer memory ---------------------
struct ExchangeView {
  int world, rank, slots;   // ranks, this rank, partials per rank per exchange
  void* peers[8];           // every rank's exchange buffer as mapped in this process
};
size_t exchange_bytes(int world, int slots, long long rows, int d);
// Merge n_groups groups of ppg chunk partials (o_in [n_groups*ppg][rows][d], lse_in) into
// slots [0, n_groups) (empty partials in [n_groups, slots)) and store them into slot `rank`
// of every rank's buffer, parity epoch & 1; then publish ready = epoch.
cudaError_t launch_merge_scatter(const ExchangeView& x, int n_groups, int ppg, long long rows, int d,
                                 const float* o_in, const float* lse_in, unsigned long long epoch, cudaStream_t st);
// Wait for every rank's slot of the epoch in this rank's buffer, merge, ack.
cudaError_t launch_gather_merge(const ExchangeView& x, long long rows, int d, unsigned long long epoch, void* out,
                                float* lse_out, cudaStream_t st);

// --- api.cu: the thread-local message read by star_last_error(); returns code ----
int set_last_error(int code, const char* msg);

// --- device error words (one per kernel file; call after synchronising) ------
cudaError_t read_and_clear_error_attn(int* code);
cudaError_t read_and_clear_error_decode(int* code);
cudaError_t read_and_clear_error_rope(int* code);
cudaError_t read_and_clear_error_merge(int* code);
cudaError_t read_and_clear_error_exchange(int* code);

// --- failure-detection test hooks (per kernel file; see common.cuh) -------------
cudaError_t set_debug_attn(unsigned long long wait_limit_ns, int flags);
cudaError_t set_debug_decode(unsigned long long wait_limit_ns, int flags);
cudaError_t set_debug_exchange(unsigned long long wait_limit_ns, int flags);

}  // namespace star
