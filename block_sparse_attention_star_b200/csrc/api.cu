// C ABI of the Star Attention hot path: argument validation, workspace
// planning and the launch sequence of each call.  See include/star.h.
#include "star.h"
#include "common.cuh"
#include "internal.h"

#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

namespace {

thread_local char g_last_error[512] = "";
thread_local cudaEvent_t g_trace_start = nullptr;
thread_local cudaEvent_t g_trace_stop = nullptr;

void trace_begin(cudaStream_t st) {
  if (g_trace_start) cudaEventRecord(g_trace_start, st);
}
void trace_end(cudaStream_t st) {
  if (g_trace_stop) cudaEventRecord(g_trace_stop, st);
}

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(STAR_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

int num_sms() { return star::current_device_sm_count(); }

int check_shape(const star_shape* s) {
  if (!s) return fail(STAR_ERR_INVALID_ARG, "shape is NULL");
  if (s->B <= 0 || s->Hq <= 0 || s->Hkv <= 0 || s->d <= 0 || s->L <= 0 || s->b <= 0 || s->n <= 0 ||
      s->T_max < 0 || s->page_tokens <= 0)
    return fail(STAR_ERR_INVALID_ARG, "shape fields must be positive (B=%d Hq=%d Hkv=%d d=%d L=%d b=%d n=%d T_max=%d P=%d)",
                s->B, s->Hq, s->Hkv, s->d, s->L, s->b, s->n, s->T_max, s->page_tokens);
  if (!(s->rope_theta > 0.0) || !std::isfinite(s->rope_theta))
    return fail(STAR_ERR_INVALID_ARG, "rope_theta must be positive and finite");
  if (s->Hq % s->Hkv) return fail(STAR_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", s->Hq, s->Hkv);
  const int G = s->Hq / s->Hkv;
  if (G != 2 && G != 4 && G != 8)
    return fail(STAR_ERR_UNSUPPORTED_SHAPE, "GQA group size Hq/Hkv = %d is not supported (2, 4 or 8)", G);
  if (s->d != 64 && s->d != 128) return fail(STAR_ERR_UNSUPPORTED_SHAPE, "head dim %d is not supported (64 or 128)", s->d);
  if ((int64_t)s->n * s->b != s->L)
    return fail(STAR_ERR_UNSUPPORTED_SHAPE,
                "L (%d) must equal n*b (%d*%d): L is the capacity; shorter contexts (a ragged last block) "
                "go through seq_len",
                s->L, s->n, s->b);
  if (s->b % 128) return fail(STAR_ERR_UNSUPPORTED_SHAPE, "block size b (%d) must be a multiple of 128", s->b);
  if (s->page_tokens % 128) return fail(STAR_ERR_UNSUPPORTED_SHAPE, "page_tokens (%d) must be a multiple of 128", s->page_tokens);
  if (s->b % s->page_tokens)
    return fail(STAR_ERR_UNSUPPORTED_SHAPE, "b (%d) must be a multiple of page_tokens (%d)", s->b, s->page_tokens);
  if (s->seq_len) {
    if (s->B > star::kMaxVarB)
      return fail(STAR_ERR_UNSUPPORTED_SHAPE, "per-sequence lengths are supported for B <= %d (B = %d)", star::kMaxVarB,
                  s->B);
    for (int i = 0; i < s->B; ++i)
      if (s->seq_len[i] < 1 || s->seq_len[i] > s->L)
        return fail(STAR_ERR_INVALID_ARG, "seq_len[%d] = %d outside [1, L = %d]", i, s->seq_len[i], s->L);
  }
  if (s->anchor < 0) return fail(STAR_ERR_INVALID_ARG, "anchor size (%d) must not be negative", s->anchor);
  if (s->anchor > s->b || s->anchor % 128)
    return fail(STAR_ERR_UNSUPPORTED_SHAPE, "anchor size (%d) must be a multiple of 128 and at most b (%d)", s->anchor,
                s->b);
  if ((int64_t)s->L + round_up(s->T_max, 128) >= (int64_t)1 << 30)
    return fail(STAR_ERR_UNSUPPORTED_SHAPE, "L + T_max too large");
  return STAR_OK;
}

int64_t pages_needed(const star_shape* s) {
  return ((int64_t)s->L + round_up(s->T_max, 128) + s->page_tokens - 1) / s->page_tokens;
}

int check_cache(const star_shape* s, const star_cache* c) {
  if (!c) return fail(STAR_ERR_INVALID_ARG, "cache is NULL");
  if (!c->k_pool || !c->v_pool || !c->page_table) return fail(STAR_ERR_INVALID_ARG, "cache pointers must be non-NULL");
  if (!aligned16(c->k_pool) || !aligned16(c->v_pool) || (reinterpret_cast<uintptr_t>(c->page_table) & 3u))
    return fail(STAR_ERR_ALIGNMENT, "cache pools must be 16-byte aligned, the page table 4-byte aligned");
  if (c->max_pages < pages_needed(s))
    return fail(STAR_ERR_CAPACITY, "page table has %d pages per sequence, %lld needed", c->max_pages,
                (long long)pages_needed(s));
  if (c->num_pages <= 0) return fail(STAR_ERR_CAPACITY, "num_pages must be positive");
  return STAR_OK;
}

star::CacheView view(const star_shape* s, const star_cache* c) {
  star::CacheView v;
  v.k_pool = c->k_pool;
  v.v_pool = c->v_pool;
  v.page_table = c->page_table;
  v.max_pages = c->max_pages;
  v.num_pages = c->num_pages;
  v.P = s->page_tokens;
  return v;
}

star::RopeTable rope_table(const star_shape* s) {
  star::RopeTable t;
  for (int j = 0; j < star::kMaxHalfDimHost; ++j)
    t.inv_freq[j] = j < s->d / 2 ? std::pow(s->rope_theta, -2.0 * j / s->d) : 0.0;
  return t;
}

float scale_log2(const star_shape* s) { return (float)(1.4426950408889634 / std::sqrt((double)s->d)); }

// Position ids and LSE values are accessed one element at a time: 4-byte alignment.
#define STAR_REQUIRE_PTR4(p, name)                                                   \
  do {                                                                               \
    if (!(p)) return fail(STAR_ERR_INVALID_ARG, "%s is NULL", name);                 \
    if (reinterpret_cast<uintptr_t>(p) & 3u)                                         \
      return fail(STAR_ERR_ALIGNMENT, "%s is not 4-byte aligned", name);             \
  } while (0)

#define STAR_REQUIRE_PTR(p, name)                                                    \
  do {                                                                               \
    if (!(p)) return fail(STAR_ERR_INVALID_ARG, "%s is NULL", name);                 \
    if (!aligned16(p)) return fail(STAR_ERR_ALIGNMENT, "%s is not 16-byte aligned", name); \
  } while (0)

// Phase 2 splits each block into chunks_per_block parts so the persistent grid
// fills the GPU with long items: the largest divisor of b/128 that keeps the item
// count within one wave (one item per SM); 1 if even that exceeds a wave.
int phase2_chunks_per_block(const star_shape* s, int T) {
  const int G = s->Hq / s->Hkv;
  int TQ = 1;
  while (TQ < T && TQ < 128) TQ <<= 1;
  const int HT = 128 / TQ;
  const int NTT = (T + TQ - 1) / TQ;
  const int NHT = (G + HT - 1) / HT;
  const int npairs = (NTT * NHT + 1) / 2;
  const int64_t base = (int64_t)s->n * s->B * s->Hkv * npairs;
  const int nb = s->b / 128;
  int best = 1;
  for (int c = 1; c <= nb; ++c)
    if (nb % c == 0 && base * c <= num_sms()) best = c;
  return best;
}

// The same choice for a shard of nblk blocks, capped so that its chunk partials never
// outnumber the whole context's (the Phase-2 workspace is sized for those).
int phase2_chunks_per_block_shard(const star_shape* s, int T, int nblk) {
  const int G = s->Hq / s->Hkv;
  int TQ = 1;
  while (TQ < T && TQ < 128) TQ <<= 1;
  const int HT = 128 / TQ;
  const int NTT = (T + TQ - 1) / TQ;
  const int NHT = (G + HT - 1) / HT;
  const int npairs = (NTT * NHT + 1) / 2;
  const int64_t base = (int64_t)nblk * s->B * s->Hkv * npairs;
  const int64_t max_parts = (int64_t)s->n * phase2_chunks_per_block(s, T);
  const int nb = s->b / 128;
  int best = 1;
  for (int c = 1; c <= nb; ++c)
    if (nb % c == 0 && base * c <= num_sms() && (int64_t)nblk * c <= max_parts) best = c;
  return best;
}

// Phase-2 scratch: RoPE(q) (bf16 [B][T][Hq][d]), then, when blocks are split into
// chunks, the chunk partials (f32 O, then LSE).
size_t phase2_q_bytes(const star_shape* s, int T) { return round_up((size_t)s->B * T * s->Hq * s->d * 2, 256); }

size_t phase2_ws_bytes(const star_shape* s, int T) {
  const int cpb = phase2_chunks_per_block(s, T);
  const size_t qb = phase2_q_bytes(s, T);
  if (cpb == 1) return qb;
  const size_t rows = (size_t)s->B * T * s->Hq;
  const size_t parts = (size_t)s->n * cpb;
  return qb + round_up(parts * rows * s->d * sizeof(float), 256) + round_up(parts * rows * sizeof(float), 256);
}

// The push variant of the Phase-2 shard always stages the chunk partials (merged into the
// exchange slots by the scatter kernel), even with one chunk per block.
size_t phase2_push_ws_bytes(const star_shape* s, int T) {
  const int cpb = phase2_chunks_per_block(s, T);
  const size_t rows = (size_t)s->B * T * s->Hq;
  const size_t parts = (size_t)s->n * cpb;
  return phase2_q_bytes(s, T) + round_up(parts * rows * s->d * sizeof(float), 256) +
         round_up(parts * rows * sizeof(float), 256);
}

int anchor_of(const star_shape* s) { return s->anchor ? s->anchor : s->b; }

// Per-sequence context lengths as shifts of the capacity frame (delta = L_s - L).
star::SeqShift shift_of(const star_shape* s) {
  star::SeqShift sh;
  memset(&sh, 0, sizeof(sh));
  sh.on = s->seq_len ? 1 : 0;
  if (sh.on)
    for (int i = 0; i < s->B; ++i) sh.delta[i] = s->seq_len[i] - s->L;
  return sh;
}

// The anchor's keys, roped at caller-given ids, per (sequence, block 2..n): bf16 [B][n-1][Hkv][a][d].
size_t anchor_ws_bytes(const star_shape* s) {
  return (size_t)s->B * (s->n - 1) * s->Hkv * anchor_of(s) * s->d * 2;
}

int decode_chunk(const star_shape* s) {
  return star::decode_pick_chunk(s->B, s->Hkv, s->Hq / s->Hkv, s->L + s->T_max, num_sms());
}

size_t decode_ws_bytes(const star_shape* s) {
  const int chunk = decode_chunk(s);
  const size_t nch = (size_t)star::decode_num_chunks(s->L + s->T_max, chunk);
  const size_t rows = (size_t)s->B * s->Hq;
  return round_up(nch * rows * s->d * sizeof(float), 256) + round_up(nch * rows * sizeof(float), 256);
}

}  // namespace

namespace star {
int set_last_error(int code, const char* msg) { return fail(code, "%s", msg); }

int current_device_sm_count() {
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64) {
    const int c = cached[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) return 148;
  if (dev >= 0 && dev < 64) cached[dev].store(sms, std::memory_order_relaxed);
  return sms;
}
}  // namespace star

extern "C" {

const char* star_version(void) { return "star-b200 0.1 (sm_100a)"; }

const char* star_last_error(void) { return g_last_error; }

int star_pages_needed(const star_shape* shape, int32_t* max_pages_out) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!max_pages_out) return fail(STAR_ERR_INVALID_ARG, "max_pages_out is NULL");
  *max_pages_out = (int32_t)pages_needed(shape);
  return STAR_OK;
}

int star_page_table_fill(const star_shape* shape, int32_t* page_table_host, int32_t max_pages, int32_t first_page) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!page_table_host) return fail(STAR_ERR_INVALID_ARG, "page_table_host is NULL");
  if (max_pages < pages_needed(shape))
    return fail(STAR_ERR_CAPACITY, "max_pages %d < %lld needed", max_pages, (long long)pages_needed(shape));
  if (first_page < 0) return fail(STAR_ERR_INVALID_ARG, "first_page must be >= 0");
  for (int64_t s = 0; s < shape->B; ++s)
    for (int64_t j = 0; j < max_pages; ++j) page_table_host[s * max_pages + j] = (int32_t)(first_page + s * max_pages + j);
  return STAR_OK;
}

int star_workspace_size(const star_shape* shape, int op, int32_t T, size_t* bytes_out) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (!bytes_out) return fail(STAR_ERR_INVALID_ARG, "bytes_out is NULL");
  switch (op) {
    case STAR_OP_PHASE1: *bytes_out = 0; return STAR_OK;
    case STAR_OP_PHASE2:
      if (T <= 0 || T > shape->T_max) return fail(STAR_ERR_INVALID_ARG, "T (%d) must be in [1, T_max=%d]", T, shape->T_max);
      *bytes_out = phase2_ws_bytes(shape, T);
      return STAR_OK;
    case STAR_OP_DECODE: *bytes_out = decode_ws_bytes(shape); return STAR_OK;
    case STAR_OP_PHASE1_ANCHOR: *bytes_out = anchor_ws_bytes(shape); return STAR_OK;
    case STAR_OP_PHASE2_PUSH:
      if (T <= 0 || T > shape->T_max) return fail(STAR_ERR_INVALID_ARG, "T (%d) must be in [1, T_max=%d]", T, shape->T_max);
      *bytes_out = phase2_push_ws_bytes(shape, T);
      return STAR_OK;
    default: return fail(STAR_ERR_INVALID_ARG, "unknown op %d", op);
  }
}

int star_build_positions(const star_shape* shape, const star_cache* cache, const int32_t* pos_ctx, int32_t* aug_pos,
                         int32_t* block_map, star_stream_t stream) {
  int rc = check_shape(shape);
  if (!rc) rc = check_cache(shape, cache);
  if (rc) return rc;
  STAR_REQUIRE_PTR4(pos_ctx, "pos_ctx");
  STAR_REQUIRE_PTR4(aug_pos, "aug_pos");
  STAR_REQUIRE_PTR4(block_map, "block_map");
  cudaError_t e = star::launch_build_positions(pos_ctx, shape->B, shape->L, shape->b, anchor_of(shape),
                                               view(shape, cache), aug_pos,
                                               block_map, (cudaStream_t)stream);
  return e == cudaSuccess ? STAR_OK : cuda_fail(e, "build_positions launch");
}

int star_kv_append(const star_shape* shape, const star_cache* cache, const void* k, const void* v, const int32_t* pos,
                   int32_t start, int32_t ntok, star_stream_t stream) {
  int rc = check_shape(shape);
  if (!rc) rc = check_cache(shape, cache);
  if (rc) return rc;
  STAR_REQUIRE_PTR(k, "k");
  STAR_REQUIRE_PTR(v, "v");
  STAR_REQUIRE_PTR4(pos, "pos");
  if (start < 0 || ntok < 0) return fail(STAR_ERR_INVALID_ARG, "start and ntok must be >= 0");
  if ((int64_t)start + ntok > (int64_t)shape->L + shape->T_max)
    return fail(STAR_ERR_CAPACITY, "slots [%d, %d) exceed L + T_max = %d", start, start + ntok, shape->L + shape->T_max);
  if (shape->seq_len && start < shape->L)
    return fail(STAR_ERR_INVALID_ARG, "with per-sequence lengths, start (%d) counts from the capacity L = %d and "
                "must be >= L", start, shape->L);
  const star::SeqShift sh = shift_of(shape);
  cudaError_t e = star::launch_rope_append(k, v, pos, shape->B, ntok, start, shape->Hkv, shape->d, view(shape, cache),
                                           rope_table(shape), (cudaStream_t)stream, &sh);
  return e == cudaSuccess ? STAR_OK : cuda_fail(e, "kv_append launch");
}

int star_phase1_encode(const star_shape* shape, const star_cache* cache, const void* q, const void* k, const void* v,
                       const int32_t* pos_ctx, void* out, void* ws, size_t ws_bytes, star_stream_t stream) {
  return star_phase1_encode_anchored(shape, cache, q, k, v, pos_ctx, nullptr, out, ws, ws_bytes, stream);
}

int star_phase1_encode_anchored(const star_shape* shape, const star_cache* cache, const void* q, const void* k,
                                const void* v, const int32_t* pos_ctx, const int32_t* anchor_pos, void* out,
                                void* ws, size_t ws_bytes, star_stream_t stream) {
  int rc = check_shape(shape);
  if (!rc) rc = check_cache(shape, cache);
  if (rc) return rc;
  STAR_REQUIRE_PTR(q, "q");
  STAR_REQUIRE_PTR(k, "k");
  STAR_REQUIRE_PTR(v, "v");
  STAR_REQUIRE_PTR4(pos_ctx, "pos_ctx");
  STAR_REQUIRE_PTR(out, "out");
  if (anchor_pos && shape->n > 1) {
    STAR_REQUIRE_PTR4(anchor_pos, "anchor_pos");
    STAR_REQUIRE_PTR(ws, "ws");
    const size_t need = anchor_ws_bytes(shape);
    if (ws_bytes < need)
      return fail(STAR_ERR_CAPACITY, "workspace %zu bytes < %zu needed for the anchor's keys", ws_bytes, need);
  }
  cudaStream_t st = (cudaStream_t)stream;
  const star::CacheView cv = view(shape, cache);
  const star::RopeTable rt = rope_table(shape);
  cudaError_t e = star::launch_rope_append(k, v, pos_ctx, shape->B, shape->L, 0, shape->Hkv, shape->d, cv, rt, st);
  if (e != cudaSuccess) return cuda_fail(e, "phase1 kv append");
  const star::SeqShift sh = shift_of(shape);
  e = star::launch_zero_slots(shape->B, shape->L, shape->L + (int)round_up(shape->T_max, 128), shape->Hkv, shape->d,
                              cv, st, &sh);
  if (e != cudaSuccess) return cuda_fail(e, "phase1 tail clear");
  const int anchor = anchor_of(shape);
  const bool own_anchor_ids = anchor_pos && shape->n > 1;
  if (own_anchor_ids) {
    e = star::launch_rope_anchor(k, anchor_pos, shape->B, shape->L, shape->n, anchor, shape->Hkv, shape->d, ws, rt, st);
    if (e != cudaSuccess) return cuda_fail(e, "phase1 anchor keys");
  }
  star::AttnLaunch a;
  memset(&a, 0, sizeof(a));
  a.mode = 0;
  a.anchor = anchor;
  a.anchor_k = own_anchor_ids ? ws : nullptr;
  a.shift = sh;
  a.B = shape->B;
  a.Hq = shape->Hq;
  a.Hkv = shape->Hkv;
  a.d = shape->d;
  a.L = shape->L;
  a.b = shape->b;
  a.n = shape->n;
  a.q = out;  // RoPE(q) is staged in the output buffer: each work item reads its Q tile, then writes O there
  a.Ntok = shape->L;
  a.cache = cv;
  a.out_bf16 = out;
  a.chunks_per_block = 1;
  a.scale_log2 = scale_log2(shape);
  const char* why = nullptr;
  trace_begin(st);
  e = star::launch_rope_q(q, pos_ctx, shape->B, shape->L, shape->Hq, shape->d, out, rt, st);
  if (e == cudaSuccess) e = star::launch_attention(a, st, &why);
  trace_end(st);
  if (e != cudaSuccess) return why ? fail(STAR_ERR_CUDA, "%s", why) : cuda_fail(e, "phase1 attention launch");
  return STAR_OK;
}

int star_encode_layers(const star_shape* shape, int32_t n_layers, const star_cache* caches, const int32_t* pos_ctx,
                       void* x, void* q, void* k, void* v, void* o, star_layer_fn fn, void* user,
                       star_stream_t stream) {
  int rc = check_shape(shape);
  if (rc) return rc;
  if (n_layers < 1) return fail(STAR_ERR_INVALID_ARG, "n_layers (%d) must be >= 1", n_layers);
  if (!caches) return fail(STAR_ERR_INVALID_ARG, "caches is NULL");
  if (!fn) return fail(STAR_ERR_INVALID_ARG, "fn is NULL");
  if (!x) return fail(STAR_ERR_INVALID_ARG, "x is NULL");
  STAR_REQUIRE_PTR(q, "q");
  STAR_REQUIRE_PTR(k, "k");
  STAR_REQUIRE_PTR(v, "v");
  STAR_REQUIRE_PTR(o, "o");
  STAR_REQUIRE_PTR4(pos_ctx, "pos_ctx");
  for (int l = 0; l < n_layers; ++l) {
    rc = check_cache(shape, &caches[l]);
    if (rc) return rc;
  }
  for (int l = 0; l < n_layers; ++l) {
    int cb = fn(l, STAR_LAYER_QKV, x, q, k, v, user, stream);
    if (cb) return fail(STAR_ERR_CALLBACK, "layer callback returned %d (layer %d, q/k/v stage)", cb, l);
    rc = star_phase1_encode(shape, &caches[l], q, k, v, pos_ctx, o, nullptr, 0, stream);
    if (rc) return rc;
    cb = fn(l, STAR_LAYER_OUT, o, x, nullptr, nullptr, user, stream);
    if (cb) return fail(STAR_ERR_CALLBACK, "layer callback returned %d (layer %d, output stage)", cb, l);
  }
  return STAR_OK;
}

int star_phase2_partial(const star_shape* shape, const star_cache* cache, const void* q, const void* k, const void* v,
                        const int32_t* q_pos, int32_t T, float* o_part, float* lse_part, void* ws, size_t ws_bytes,
                        star_stream_t stream) {
  int rc = check_shape(shape);
  if (!rc) rc = check_cache(shape, cache);
  if (rc) return rc;
  STAR_REQUIRE_PTR(q, "q");
  STAR_REQUIRE_PTR4(q_pos, "q_pos");
  STAR_REQUIRE_PTR(o_part, "o_part");
  STAR_REQUIRE_PTR4(lse_part, "lse_part");
  if ((k == nullptr) != (v == nullptr)) return fail(STAR_ERR_INVALID_ARG, "k and v must both be given or both be NULL");
  if (T <= 0 || T > shape->T_max) return fail(STAR_ERR_INVALID_ARG, "T (%d) must be in [1, T_max=%d]", T, shape->T_max);
  const size_t need = phase2_ws_bytes(shape, T);
  STAR_REQUIRE_PTR(ws, "ws");
  if (ws_bytes < need) return fail(STAR_ERR_CAPACITY, "workspace %zu bytes < %zu needed", ws_bytes, need);
  cudaStream_t st = (cudaStream_t)stream;
  const star::CacheView cv = view(shape, cache);
  const star::RopeTable rt = rope_table(shape);
  if (k) {
    STAR_REQUIRE_PTR(k, "k");
    STAR_REQUIRE_PTR(v, "v");
    const star::SeqShift shq = shift_of(shape);
    cudaError_t e = star::launch_rope_append(k, v, q_pos, shape->B, T, shape->L, shape->Hkv, shape->d, cv, rt, st, &shq);
    if (e != cudaSuccess) return cuda_fail(e, "phase2 kv append");
  }
  const int cpb = phase2_chunks_per_block(shape, T);
  const size_t rows = (size_t)shape->B * T * shape->Hq;
  const size_t parts = (size_t)shape->n * cpb;
  void* q_rot = ws;
  char* chunk_ws = reinterpret_cast<char*>(ws) + phase2_q_bytes(shape, T);
  float* o_dst = o_part;
  float* l_dst = lse_part;
  if (cpb > 1) {
    o_dst = reinterpret_cast<float*>(chunk_ws);
    l_dst = reinterpret_cast<float*>(chunk_ws + round_up(parts * rows * shape->d * sizeof(float), 256));
  }
  star::AttnLaunch a;
  memset(&a, 0, sizeof(a));
  a.mode = 1;
  a.shift = shift_of(shape);
  a.B = shape->B;
  a.Hq = shape->Hq;
  a.Hkv = shape->Hkv;
  a.d = shape->d;
  a.L = shape->L;
  a.b = shape->b;
  a.n = shape->n;
  a.q = q_rot;
  a.Ntok = T;
  a.cache = cv;
  a.out_f32 = o_dst;
  a.lse_f32 = l_dst;
  a.chunks_per_block = cpb;
  a.scale_log2 = scale_log2(shape);
  const char* why = nullptr;
  trace_begin(st);
  cudaError_t e = star::launch_rope_q(q, q_pos, shape->B, T, shape->Hq, shape->d, q_rot, rt, st);
  if (e == cudaSuccess) e = star::launch_attention(a, st, &why);
  trace_end(st);
  if (e != cudaSuccess) return why ? fail(STAR_ERR_CUDA, "%s", why) : cuda_fail(e, "phase2 attention launch");
  if (cpb > 1) {
    e = star::launch_lse_merge(shape->n, cpb, (int64_t)rows, shape->d, o_dst, l_dst, o_part, false, lse_part, st);
    if (e != cudaSuccess) return cuda_fail(e, "phase2 chunk merge");
  }
  return STAR_OK;
}

int star_lse_merge(int32_t n_parts, int64_t rows, int32_t d, const float* o_part, const float* lse_part, void* out,
                   float* lse_out, star_stream_t stream) {
  if (n_parts <= 0 || rows < 0) return fail(STAR_ERR_INVALID_ARG, "n_parts must be > 0 and rows >= 0");
  if (d != 64 && d != 128) return fail(STAR_ERR_UNSUPPORTED_SHAPE, "head dim %d is not supported (64 or 128)", d);
  STAR_REQUIRE_PTR(o_part, "o_part");
  STAR_REQUIRE_PTR4(lse_part, "lse_part");
  STAR_REQUIRE_PTR(out, "out");
  if (lse_out && (reinterpret_cast<uintptr_t>(lse_out) & 3u)) return fail(STAR_ERR_ALIGNMENT, "lse_out is not 4-byte aligned");
  cudaError_t e = star::launch_lse_merge(1, n_parts, rows, d, o_part, lse_part, out, true, lse_out, (cudaStream_t)stream);
  return e == cudaSuccess ? STAR_OK : cuda_fail(e, "lse_merge launch");
}

int star_decode_step(const star_shape* shape, const star_cache* cache, const void* q, const void* k, const void* v,
                     const int32_t* pos, int32_t cur_len, void* out, float* lse_out, void* ws, size_t ws_bytes,
                     star_stream_t stream) {
  int rc = check_shape(shape);
  if (!rc) rc = check_cache(shape, cache);
  if (rc) return rc;
  STAR_REQUIRE_PTR(q, "q");
  STAR_REQUIRE_PTR(k, "k");
  STAR_REQUIRE_PTR(v, "v");
  STAR_REQUIRE_PTR4(pos, "pos");
  STAR_REQUIRE_PTR(out, "out");
  STAR_REQUIRE_PTR(ws, "ws");
  if (lse_out && (reinterpret_cast<uintptr_t>(lse_out) & 3u)) return fail(STAR_ERR_ALIGNMENT, "lse_out is not 4-byte aligned");
  if (cur_len < 0 || cur_len >= shape->L + shape->T_max)
    return fail(STAR_ERR_CAPACITY, "cur_len %d outside [0, L + T_max = %d)", cur_len, shape->L + shape->T_max);
  if (shape->seq_len && cur_len < shape->L)
    return fail(STAR_ERR_INVALID_ARG, "with per-sequence lengths, cur_len (%d) counts from the capacity L = %d and "
                "must be >= L", cur_len, shape->L);
  const size_t need = decode_ws_bytes(shape);
  if (ws_bytes < need) return fail(STAR_ERR_CAPACITY, "workspace %zu bytes < %zu needed", ws_bytes, need);
  cudaStream_t st = (cudaStream_t)stream;
  const star::CacheView cv = view(shape, cache);
  const star::RopeTable rt = rope_table(shape);
  cudaError_t e;
  // The workspace holds the chunks of the capacity at the capacity's chunk; per-sequence
  // lengths may take a longer chunk (never a shorter one) to balance the real work.
  const int chunk_cap = decode_chunk(shape);
  const int n_keys = cur_len + 1;
  int chunk = chunk_cap;
  if (shape->seq_len) {
    int keys_of[star::kMaxVarB];
    for (int s = 0; s < shape->B; ++s) keys_of[s] = n_keys + shape->seq_len[s] - shape->L;
    chunk = star::decode_pick_chunk_var(shape->B, shape->Hkv, keys_of, chunk_cap, num_sms());
  }
  const int nch = star::decode_num_chunks(n_keys, chunk);
  const size_t rows = (size_t)shape->B * shape->Hq;
  const size_t nch_max = (size_t)star::decode_num_chunks(shape->L + shape->T_max, chunk_cap);
  star::DecodeLaunch a;
  a.B = shape->B;
  a.Hq = shape->Hq;
  a.Hkv = shape->Hkv;
  a.d = shape->d;
  a.q = q;
  a.k_new = k;
  a.v_new = v;
  a.pos = pos;
  a.n_keys = n_keys;
  a.k_lo = 0;
  a.append = 1;
  a.shift = shift_of(shape);
  a.chunk = chunk;
  a.cache = cv;
  a.o_ws = reinterpret_cast<float*>(ws);
  a.lse_ws = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + round_up(nch_max * rows * shape->d * sizeof(float), 256));
  a.scale_log2 = scale_log2(shape);
  a.rope = rt;
  trace_begin(st);
  e = star::launch_decode(a, st);
  trace_end(st);
  if (e != cudaSuccess) return cuda_fail(e, "decode attention launch");
  e = star::launch_lse_merge(1, nch, (int64_t)rows, shape->d, a.o_ws, a.lse_ws, out, true, lse_out, st);
  return e == cudaSuccess ? STAR_OK : cuda_fail(e, "decode merge launch");
}

// ---------------------------------------------------------------------------
// Shards: a contiguous block range per GPU
// ---------------------------------------------------------------------------
static int check_shard(const star_shape* s, const star_shard* sh) {
  if (!sh) return fail(STAR_ERR_INVALID_ARG, "shard is NULL");
  if (sh->block_begin < 0 || sh->block_end <= sh->block_begin || sh->block_end > s->n)
    return fail(STAR_ERR_INVALID_ARG, "shard blocks [%d, %d) outside [0, n = %d)", sh->block_begin, sh->block_end, s->n);
  if (s->seq_len) return fail(STAR_ERR_UNSUPPORTED_SHAPE, "shards need sequences of one length (seq_len must be NULL)");
  return STAR_OK;
}

int star_phase1_encode_shard(const star_shape* shape, const star_cache* cache, const star_shard* shard, const void* q,
                             const void* k, const void* v, const int32_t* pos, const void* k_anchor,
                             const void* v_anchor, const int32_t* pos_anchor, void* out, star_stream_t stream) {
  int rc = check_shape(shape);
  if (!rc) rc = check_cache(shape, cache);
  if (!rc) rc = check_shard(shape, shard);
  if (rc) return rc;
  STAR_REQUIRE_PTR(q, "q");
  STAR_REQUIRE_PTR(k, "k");
  STAR_REQUIRE_PTR(v, "v");
  STAR_REQUIRE_PTR4(pos, "pos");
  STAR_REQUIRE_PTR(out, "out");
  const int i0 = shard->block_begin, nblk = shard->block_end - shard->block_begin;
  const int anchor = anchor_of(shape);
  if (i0 > 0) {
    STAR_REQUIRE_PTR(k_anchor, "k_anchor");
    STAR_REQUIRE_PTR(v_anchor, "v_anchor");
    STAR_REQUIRE_PTR4(pos_anchor, "pos_anchor");
  }
  cudaStream_t st = (cudaStream_t)stream;
  const star::CacheView cv = view(shape, cache);
  const star::RopeTable rt = rope_table(shape);
  // The range's own tokens at their cache slots, and the anchor (block 1's first a tokens,
  // read by every later block) when the range does not hold block 1.
  cudaError_t e = star::launch_rope_append(k, v, pos, shape->B, nblk * shape->b, i0 * shape->b, shape->Hkv, shape->d,
                                           cv, rt, st);
  if (e == cudaSuccess && i0 > 0)
    e = star::launch_rope_append(k_anchor, v_anchor, pos_anchor, shape->B, anchor, 0, shape->Hkv, shape->d, cv, rt, st);
  if (e == cudaSuccess && shard->block_end == shape->n)
    e = star::launch_zero_slots(shape->B, shape->L, shape->L + (int)round_up(shape->T_max, 128), shape->Hkv, shape->d,
                                cv, st);
  if (e != cudaSuccess) return cuda_fail(e, "phase1 shard kv append");
  star::AttnLaunch a;
  memset(&a, 0, sizeof(a));
  a.mode = 0;
  a.anchor = anchor;
  a.B = shape->B;
  a.Hq = shape->Hq;
  a.Hkv = shape->Hkv;
  a.d = shape->d;
  a.L = shape->L;
  a.b = shape->b;
  a.n = shape->n;
  a.q = out;
  a.Ntok = shape->L;
  a.cache = cv;
  a.out_bf16 = out;
  a.chunks_per_block = 1;
  a.scale_log2 = scale_log2(shape);
  a.blk0 = i0;
  a.nblk = nblk;
  const char* why = nullptr;
  trace_begin(st);
  e = star::launch_rope_q(q, pos, shape->B, nblk * shape->b, shape->Hq, shape->d, out, rt, st);
  if (e == cudaSuccess) e = star::launch_attention(a, st, &why);
  trace_end(st);
  if (e != cudaSuccess) return why ? fail(STAR_ERR_CUDA, "%s", why) : cuda_fail(e, "phase1 shard attention launch");
  return STAR_OK;
}

static int check_exchange(const star_exchange* ex, int min_slots) {
  if (!ex) return fail(STAR_ERR_INVALID_ARG, "exchange is NULL");
  if (ex->world < 1 || ex->world > 8) return fail(STAR_ERR_UNSUPPORTED_SHAPE, "exchange world %d outside [1, 8]", ex->world);
  if (ex->rank < 0 || ex->rank >= ex->world)
    return fail(STAR_ERR_INVALID_ARG, "exchange rank %d outside [0, %d)", ex->rank, ex->world);
  if (ex->slots < min_slots || ex->slots < 1)
    return fail(STAR_ERR_CAPACITY, "exchange holds %d partials per rank, %d needed", ex->slots, min_slots);
  for (int w = 0; w < ex->world; ++w) {
    if (!ex->peers[w]) return fail(STAR_ERR_INVALID_ARG, "exchange peers[%d] is NULL", w);
    if (reinterpret_cast<uintptr_t>(ex->peers[w]) & 255u)
      return fail(STAR_ERR_ALIGNMENT, "exchange peers[%d] is not 256-byte aligned", w);
  }
  return STAR_OK;
}

static star::ExchangeView exchange_view(const star_exchange* ex) {
  star::ExchangeView x;
  memset(&x, 0, sizeof(x));
  x.world = ex->world;
  x.rank = ex->rank;
  x.slots = ex->slots;
  for (int w = 0; w < ex->world; ++w) x.peers[w] = ex->peers[w];
  return x;
}

// Phase-2 partials of a shard; ex == NULL: into o_part / lse_part, else pushed into the
// exchange slots of every rank (epoch).
static int phase2_shard(const star_shape* shape, const star_cache* cache, const star_shard* shard, const void* q,
                        const void* k, const void* v, const int32_t* q_pos, int32_t T, float* o_part, float* lse_part,
                        const star_exchange* ex, uint64_t epoch, void* ws, size_t ws_bytes, star_stream_t stream) {
  int rc = check_shape(shape);
  if (!rc) rc = check_cache(shape, cache);
  if (!rc) rc = check_shard(shape, shard);
  if (!rc && ex) rc = check_exchange(ex, shard->block_end - shard->block_begin);
  if (rc) return rc;
  STAR_REQUIRE_PTR(q, "q");
  STAR_REQUIRE_PTR4(q_pos, "q_pos");
  if (!ex) {
    STAR_REQUIRE_PTR(o_part, "o_part");
    STAR_REQUIRE_PTR4(lse_part, "lse_part");
  } else if (epoch == 0) {
    return fail(STAR_ERR_INVALID_ARG, "exchange epochs start at 1");
  }
  if ((k == nullptr) != (v == nullptr)) return fail(STAR_ERR_INVALID_ARG, "k and v must both be given or both be NULL");
  if (T <= 0 || T > shape->T_max) return fail(STAR_ERR_INVALID_ARG, "T (%d) must be in [1, T_max=%d]", T, shape->T_max);
  const bool tail = shard->block_end == shape->n;
  if (k && !tail) return fail(STAR_ERR_INVALID_ARG, "only the shard holding the last block appends the query's k, v");
  const size_t need = ex ? phase2_push_ws_bytes(shape, T) : phase2_ws_bytes(shape, T);
  STAR_REQUIRE_PTR(ws, "ws");
  if (ws_bytes < need) return fail(STAR_ERR_CAPACITY, "workspace %zu bytes < %zu needed", ws_bytes, need);
  cudaStream_t st = (cudaStream_t)stream;
  const star::CacheView cv = view(shape, cache);
  const star::RopeTable rt = rope_table(shape);
  if (k) {
    STAR_REQUIRE_PTR(k, "k");
    STAR_REQUIRE_PTR(v, "v");
    cudaError_t e = star::launch_rope_append(k, v, q_pos, shape->B, T, shape->L, shape->Hkv, shape->d, cv, rt, st);
    if (e != cudaSuccess) return cuda_fail(e, "phase2 shard kv append");
  }
  const int nblk = shard->block_end - shard->block_begin;
  const int cpb = phase2_chunks_per_block_shard(shape, T, nblk);
  const size_t rows = (size_t)shape->B * T * shape->Hq;
  const size_t parts = (size_t)nblk * cpb;
  void* q_rot = ws;
  char* chunk_ws = reinterpret_cast<char*>(ws) + phase2_q_bytes(shape, T);
  float* o_dst = o_part;
  float* l_dst = lse_part;
  if (cpb > 1 || ex) {
    o_dst = reinterpret_cast<float*>(chunk_ws);
    l_dst = reinterpret_cast<float*>(chunk_ws + round_up(parts * rows * shape->d * sizeof(float), 256));
  }
  star::AttnLaunch a;
  memset(&a, 0, sizeof(a));
  a.mode = 1;
  a.B = shape->B;
  a.Hq = shape->Hq;
  a.Hkv = shape->Hkv;
  a.d = shape->d;
  a.L = shape->L;
  a.b = shape->b;
  a.n = shape->n;
  a.q = q_rot;
  a.Ntok = T;
  a.cache = cv;
  a.out_f32 = o_dst;
  a.lse_f32 = l_dst;
  a.chunks_per_block = cpb;
  a.scale_log2 = scale_log2(shape);
  a.blk0 = shard->block_begin;
  a.nblk = nblk;
  a.no_tail = tail ? 0 : 1;
  const char* why = nullptr;
  trace_begin(st);
  cudaError_t e = star::launch_rope_q(q, q_pos, shape->B, T, shape->Hq, shape->d, q_rot, rt, st);
  if (e == cudaSuccess) e = star::launch_attention(a, st, &why);
  trace_end(st);
  if (e != cudaSuccess) return why ? fail(STAR_ERR_CUDA, "%s", why) : cuda_fail(e, "phase2 shard attention launch");
  if (ex) {
    e = star::launch_merge_scatter(exchange_view(ex), nblk, cpb, (long long)rows, shape->d, o_dst, l_dst,
                                   (unsigned long long)epoch, st);
    if (e != cudaSuccess) return cuda_fail(e, "phase2 shard push");
  } else if (cpb > 1) {
    e = star::launch_lse_merge(nblk, cpb, (int64_t)rows, shape->d, o_dst, l_dst, o_part, false, lse_part, st);
    if (e != cudaSuccess) return cuda_fail(e, "phase2 shard chunk merge");
  }
  return STAR_OK;
}

int star_phase2_partial_shard(const star_shape* shape, const star_cache* cache, const star_shard* shard, const void* q,
                              const void* k, const void* v, const int32_t* q_pos, int32_t T, float* o_part,
                              float* lse_part, void* ws, size_t ws_bytes, star_stream_t stream) {
  return phase2_shard(shape, cache, shard, q, k, v, q_pos, T, o_part, lse_part, nullptr, 0, ws, ws_bytes, stream);
}

int star_phase2_partial_shard_push(const star_shape* shape, const star_cache* cache, const star_shard* shard,
                                   const void* q, const void* k, const void* v, const int32_t* q_pos, int32_t T,
                                   const star_exchange* ex, uint64_t epoch, void* ws, size_t ws_bytes,
                                   star_stream_t stream) {
  if (!ex) return fail(STAR_ERR_INVALID_ARG, "exchange is NULL");
  return phase2_shard(shape, cache, shard, q, k, v, q_pos, T, nullptr, nullptr, ex, epoch, ws, ws_bytes, stream);
}

static int decode_shard(const star_shape* shape, const star_cache* cache, const star_shard* shard, const void* q,
                        const void* k, const void* v, const int32_t* pos, int32_t cur_len, float* o_part,
                        float* lse_part, const star_exchange* ex, uint64_t epoch, void* ws, size_t ws_bytes,
                        star_stream_t stream) {
  int rc = check_shape(shape);
  if (!rc) rc = check_cache(shape, cache);
  if (!rc) rc = check_shard(shape, shard);
  if (!rc && ex) rc = check_exchange(ex, 1);
  if (rc) return rc;
  STAR_REQUIRE_PTR(q, "q");
  if (!ex) {
    STAR_REQUIRE_PTR4(o_part, "o_part");
    STAR_REQUIRE_PTR4(lse_part, "lse_part");
  } else if (epoch == 0) {
    return fail(STAR_ERR_INVALID_ARG, "exchange epochs start at 1");
  }
  STAR_REQUIRE_PTR(ws, "ws");
  const bool tail = shard->block_end == shape->n;
  if (tail) {
    STAR_REQUIRE_PTR(k, "k");
    STAR_REQUIRE_PTR(v, "v");
    STAR_REQUIRE_PTR4(pos, "pos");
    if (cur_len < shape->L || cur_len >= shape->L + shape->T_max)
      return fail(STAR_ERR_CAPACITY, "cur_len %d outside [L = %d, L + T_max = %d)", cur_len, shape->L,
                  shape->L + shape->T_max);
  } else {
    STAR_REQUIRE_PTR4(pos, "pos");
  }
  const size_t need = decode_ws_bytes(shape);
  if (ws_bytes < need) return fail(STAR_ERR_CAPACITY, "workspace %zu bytes < %zu needed", ws_bytes, need);
  cudaStream_t st = (cudaStream_t)stream;
  // Keys of the range: its blocks' context keys, plus the tail up to the new token (appended
  // here) on the shard that holds the last block.
  const int k_lo = shard->block_begin * shape->b;
  const int n_keys = tail ? cur_len + 1 : shard->block_end * shape->b;
  const int chunk_cap = decode_chunk(shape);
  const size_t nch_max = (size_t)star::decode_num_chunks(shape->L + shape->T_max, chunk_cap);
  int chunk = star::decode_pick_chunk(shape->B, shape->Hkv, shape->Hq / shape->Hkv, n_keys - k_lo, num_sms());
  while ((size_t)star::decode_num_chunks(n_keys - k_lo, chunk) > nch_max) chunk += 128;  // fits the workspace
  const int nch = star::decode_num_chunks(n_keys - k_lo, chunk);
  const size_t rows = (size_t)shape->B * shape->Hq;
  star::DecodeLaunch a;
  memset(&a, 0, sizeof(a));
  a.B = shape->B;
  a.Hq = shape->Hq;
  a.Hkv = shape->Hkv;
  a.d = shape->d;
  a.q = q;
  a.k_new = tail ? k : q;  // read only by the CTA that appends (tail shard)
  a.v_new = tail ? v : q;
  a.pos = pos;
  a.n_keys = n_keys;
  a.k_lo = k_lo;
  a.append = tail ? 1 : 0;
  a.chunk = chunk;
  a.cache = view(shape, cache);
  a.o_ws = reinterpret_cast<float*>(ws);
  a.lse_ws = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + round_up(nch_max * rows * shape->d * sizeof(float), 256));
  a.scale_log2 = scale_log2(shape);
  a.rope = rope_table(shape);
  trace_begin(st);
  cudaError_t e = star::launch_decode(a, st);
  trace_end(st);
  if (e != cudaSuccess) return cuda_fail(e, "decode shard launch");
  if (ex) {
    e = star::launch_merge_scatter(exchange_view(ex), 1, nch, (long long)rows, shape->d, a.o_ws, a.lse_ws,
                                   (unsigned long long)epoch, st);
    return e == cudaSuccess ? STAR_OK : cuda_fail(e, "decode shard push");
  }
  e = star::launch_lse_merge(1, nch, (int64_t)rows, shape->d, a.o_ws, a.lse_ws, o_part, false, lse_part, st);
  return e == cudaSuccess ? STAR_OK : cuda_fail(e, "decode shard merge launch");
}

int star_decode_partial_shard(const star_shape* shape, const star_cache* cache, const star_shard* shard, const void* q,
                              const void* k, const void* v, const int32_t* pos, int32_t cur_len, float* o_part,
                              float* lse_part, void* ws, size_t ws_bytes, star_stream_t stream) {
  return decode_shard(shape, cache, shard, q, k, v, pos, cur_len, o_part, lse_part, nullptr, 0, ws, ws_bytes, stream);
}

int star_decode_partial_shard_push(const star_shape* shape, const star_cache* cache, const star_shard* shard,
                                   const void* q, const void* k, const void* v, const int32_t* pos, int32_t cur_len,
                                   const star_exchange* ex, uint64_t epoch, void* ws, size_t ws_bytes,
                                   star_stream_t stream) {
  if (!ex) return fail(STAR_ERR_INVALID_ARG, "exchange is NULL");
  return decode_shard(shape, cache, shard, q, k, v, pos, cur_len, nullptr, nullptr, ex, epoch, ws, ws_bytes, stream);
}

int star_exchange_size(int32_t world, int32_t slots, int64_t rows, int32_t d, size_t* bytes_out) {
  if (!bytes_out) return fail(STAR_ERR_INVALID_ARG, "bytes_out is NULL");
  if (world < 1 || world > 8) return fail(STAR_ERR_UNSUPPORTED_SHAPE, "exchange world %d outside [1, 8]", world);
  if (slots < 1 || rows < 1) return fail(STAR_ERR_INVALID_ARG, "slots and rows must be positive");
  if (d != 64 && d != 128) return fail(STAR_ERR_UNSUPPORTED_SHAPE, "head dim %d is not supported (64 or 128)", d);
  *bytes_out = star::exchange_bytes(world, slots, (long long)rows, d);
  return STAR_OK;
}

int star_exchange_merge(const star_exchange* ex, int64_t rows, int32_t d, uint64_t epoch, void* out, float* lse_out,
                        star_stream_t stream) {
  int rc = check_exchange(ex, 1);
  if (rc) return rc;
  if (rows < 1) return fail(STAR_ERR_INVALID_ARG, "rows must be positive");
  if (d != 64 && d != 128) return fail(STAR_ERR_UNSUPPORTED_SHAPE, "head dim %d is not supported (64 or 128)", d);
  if (epoch == 0) return fail(STAR_ERR_INVALID_ARG, "exchange epochs start at 1");
  STAR_REQUIRE_PTR(out, "out");
  if (lse_out && (reinterpret_cast<uintptr_t>(lse_out) & 3u)) return fail(STAR_ERR_ALIGNMENT, "lse_out is not 4-byte aligned");
  cudaError_t e = star::launch_gather_merge(exchange_view(ex), (long long)rows, d, (unsigned long long)epoch, out,
                                            lse_out, (cudaStream_t)stream);
  return e == cudaSuccess ? STAR_OK : cuda_fail(e, "exchange merge launch");
}

typedef CUresult (*GetAddressRangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);

int star_ipc_export(const void* ptr, void* handle_out, uint64_t* offset_out) {
  if (!ptr || !handle_out || !offset_out) return fail(STAR_ERR_INVALID_ARG, "NULL argument");
  static GetAddressRangeFn range = nullptr;
  if (!range) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return fail(STAR_ERR_CUDA, "cuMemGetAddressRange is not available");
    range = reinterpret_cast<GetAddressRangeFn>(fn);
  }
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range(&base, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS)
    return fail(STAR_ERR_INVALID_ARG, "pointer is not device memory of this process");
  cudaIpcMemHandle_t h;
  cudaError_t e = cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base));
  if (e != cudaSuccess) return cuda_fail(e, "cudaIpcGetMemHandle");
  static_assert(sizeof(h) == 64, "IPC handle size");
  memcpy(handle_out, &h, sizeof(h));
  *offset_out = (uint64_t)(reinterpret_cast<CUdeviceptr>(ptr) - base);
  return STAR_OK;
}

int star_ipc_open(const void* handle, uint64_t offset, void** ptr_out) {
  if (!handle || !ptr_out) return fail(STAR_ERR_INVALID_ARG, "NULL argument");
  cudaIpcMemHandle_t h;
  memcpy(&h, handle, sizeof(h));
  void* base = nullptr;
  cudaError_t e = cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess);
  if (e != cudaSuccess) return cuda_fail(e, "cudaIpcOpenMemHandle");
  *ptr_out = reinterpret_cast<char*>(base) + offset;
  return STAR_OK;
}

int star_ipc_close(void* ptr, uint64_t offset) {
  if (!ptr) return fail(STAR_ERR_INVALID_ARG, "ptr is NULL");
  cudaError_t e = cudaIpcCloseMemHandle(reinterpret_cast<char*>(ptr) - offset);
  return e == cudaSuccess ? STAR_OK : cuda_fail(e, "cudaIpcCloseMemHandle");
}

int star_set_trace_events(void* start_event, void* stop_event) {
  if ((start_event == nullptr) != (stop_event == nullptr))
    return fail(STAR_ERR_INVALID_ARG, "trace events must both be given or both be NULL");
  g_trace_start = reinterpret_cast<cudaEvent_t>(start_event);
  g_trace_stop = reinterpret_cast<cudaEvent_t>(stop_event);
  return STAR_OK;
}

int star_device_status(star_stream_t stream, int32_t* status_out) {
  int code = 0;
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  cudaError_t (*readers[])(int*) = {star::read_and_clear_error_attn, star::read_and_clear_error_decode,
                                   star::read_and_clear_error_rope, star::read_and_clear_error_merge,
                                   star::read_and_clear_error_exchange};
  for (auto rd : readers) {
    if (e != cudaSuccess) break;
    int c = 0;
    e = rd(&c);
    if (code == 0) code = c;
  }
  if (status_out) *status_out = code;
  if (e != cudaSuccess) return cuda_fail(e, "device status");
  if (code == star::kDevBadPage) return fail(STAR_ERR_CAPACITY, "a page-table entry was outside [0, num_pages)");
  if (code == star::kDevBadPartial)
    return fail(STAR_ERR_INVALID_ARG, "a merged partial had a NaN or +inf log-sum-exp (it was skipped)");
  if (code != 0) return fail(STAR_ERR_TIMEOUT, "a kernel gave up a bounded wait (code %d)", code);
  return STAR_OK;
}

int star_debug_set(uint64_t wait_limit_ns, int32_t flags) {
  if (flags & ~STAR_DEBUG_SKIP_FIRST_LOAD) return fail(STAR_ERR_INVALID_ARG, "unknown debug flags 0x%x", flags);
  const unsigned long long limit = wait_limit_ns ? wait_limit_ns : star::kDefaultWaitLimitNs;
  const int dev_flags = (flags & STAR_DEBUG_SKIP_FIRST_LOAD) ? star::kDebugSkipFirstLoad : 0;
  cudaError_t e = star::set_debug_attn(limit, dev_flags);
  if (e == cudaSuccess) e = star::set_debug_decode(limit, dev_flags);
  if (e == cudaSuccess) e = star::set_debug_exchange(limit, 0);
  return e == cudaSuccess ? STAR_OK : cuda_fail(e, "debug settings");
}

}  // extern "C"
