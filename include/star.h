/*
 * star.h -- C ABI of the Star Attention hot path on NVIDIA B200 (sm_100a).
 *
 * Star Attention ("Star Attention: Efficient LLM Inference over Long
 * Sequences"; walk-through in "Star Attention 完全拆解(一):锚点块、分块上下文编码
 * 与两阶段全局注意力") is a two-phase block-sparse approximation of attention:
 *
 *   Phase 1 (context encoding): the context c = [c_1 .. c_n] of L = n*b tokens is
 *     split into blocks of b tokens; every block after the first is prefixed by
 *     the anchor block c_1, which keeps its own position ids, and runs causal
 *     attention locally; the anchor's KV is discarded and only c_i's is cached.
 *   Phase 2 (query and generation): query and generated tokens attend to every
 *     cached block; each block yields a local (output, log-sum-exp) pair and the
 *     pairs are merged exactly into global attention.
 *
 * Conventions for every call below
 *   - One attention layer.  Q, K, V are that layer's projections (pre-RoPE).
 *   - Tensor pointers are DEVICE pointers owned by the caller, contiguous,
 *     16-byte aligned (position-id arrays, LSE arrays and the page table: 4-byte
 *     aligned); bf16 means IEEE bfloat16.  Layout is [B, tokens, heads, d]
 *     ("bshd") unless stated.  Position ids are int32.
 *   - The library allocates no device memory.  Scratch space is passed in as
 *     `ws` of at least star_workspace_size() bytes.
 *   - Every call is asynchronous on the caller's CUDA stream `stream` (a
 *     cudaStream_t; NULL = legacy default stream) and never synchronises, except
 *     star_device_status().  The compute calls can be captured into a CUDA graph
 *     once each has run eagerly on the device (the first call of a kernel sets its
 *     shared-memory opt-in); a replay recomputes from the buffers' current contents.
 *   - Return value: STAR_OK (0) or a negative STAR_ERR_* code; star_last_error()
 *     then describes the failure (thread-local).  Arguments are validated on the
 *     host before anything is launched; a failing call launches nothing.
 *   - RoPE: rotate-half pairing (x_j, x_{j+d/2}), inv_freq_j = theta^(-2j/d),
 *     angle pos * inv_freq_j formed in float64; rotated Q and K are rounded to
 *     bf16.  Softmax scale 1/sqrt(d).  GQA: query head h uses KV head h / (Hq/Hkv).
 *   - LSE values are natural logarithms: log sum_k exp(q.k / sqrt(d)).
 */
#ifndef STAR_H_
#define STAR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* star_stream_t; /* == cudaStream_t */

enum {
  STAR_OK = 0,
  STAR_ERR_INVALID_ARG = -1,      /* null pointer, negative size, inconsistent shape */
  STAR_ERR_UNSUPPORTED_SHAPE = -2,/* valid but not supported: d not in {64,128}, odd Hq/Hkv, L != n*b, ... */
  STAR_ERR_ALIGNMENT = -3,        /* a pointer is not aligned as stated above */
  STAR_ERR_CAPACITY = -4,         /* page table / pool / workspace too small */
  STAR_ERR_CUDA = -5,             /* a CUDA runtime or driver call failed */
  STAR_ERR_TIMEOUT = -6,          /* a kernel gave up a bounded wait (see star_device_status) */
  STAR_ERR_CALLBACK = -7          /* a caller callback returned non-zero (star_encode_layers) */
};

/* Workspace query selectors. */
enum { STAR_OP_PHASE1 = 1, STAR_OP_PHASE2 = 2, STAR_OP_DECODE = 3, STAR_OP_PHASE1_ANCHOR = 4, STAR_OP_PHASE2_PUSH = 5 };

/* Problem shape ("问题定义与记号": context c of n blocks of b tokens, query q). */
typedef struct star_shape {
  int32_t B;           /* independent sequences */
  int32_t Hq;          /* query heads; Hq / Hkv must be even (2, 4, 8) */
  int32_t Hkv;         /* key/value heads */
  int32_t d;           /* head dim: 64 or 128 */
  int32_t L;           /* context tokens, L = n * b */
  int32_t b;           /* block size; multiple of 128 and of page_tokens */
  int32_t n;           /* number of blocks */
  int32_t T_max;       /* tail capacity after the context: query + generated tokens */
  int32_t page_tokens; /* P: tokens per cache page; multiple of 128 */
  double rope_theta;   /* RoPE base, e.g. 500000 */
  int32_t anchor;      /* anchor size a: the first a tokens of block 1 ("仓库里的真实实现":
                          anchor_block_size is a parameter of its own); 0 means b (the pages'
                          default, the whole first block); a multiple of 128 and <= b */
  const int32_t* seq_len; /* HOST int32 [B] or NULL: per-sequence context lengths L_s, 1 <= L_s <= L
                          (B <= 256).  L is then the capacity (a multiple of b); sequence s has
                          ceil(L_s / b) blocks, the last one ragged ("问题定义与记号" splits the
                          context into blocks of b tokens; an uneven split ends in a short
                          block), and its tail (query and generated tokens) starts at L_s.
                          Context arrays stay padded to L; rows >= L_s of outputs are
                          unspecified.  Cache indices given to star_kv_append (start) and
                          star_decode_step (cur_len) are in the frame of a sequence of length
                          L: sequence s uses index + L_s - L, so they must be >= L.
                          Phase-2 partials of blocks a sequence does not have are empty
                          (O = 0, LSE = -inf), which star_lse_merge skips. */
} star_shape;

/* Paged KV cache ("局部注意力与 KV 丢弃": only non-anchor KV is kept).
 * k_pool, v_pool: bf16 [num_pages][Hkv][page_tokens][d]; one (page, head) run is
 * page_tokens*d*2 contiguous bytes.  Token t of sequence s lives in physical page
 * page_table[s*max_pages + t/page_tokens], slot t % page_tokens; K is stored
 * after RoPE, V as given.  page_table is a DEVICE int32 array [B][max_pages]
 * that the caller fills (star_page_table_fill gives the block-contiguous one:
 * block i of a sequence occupies consecutive physical pages).  It must cover
 * tokens [0, L + round_up(T_max, 128)). */
typedef struct star_cache {
  void* k_pool;
  void* v_pool;
  const int32_t* page_table;
  int32_t max_pages;   /* logical pages per sequence */
  int32_t num_pages;   /* physical pages in each pool */
} star_cache;

/* Library version string (static storage). */
const char* star_version(void);

/* Message of the last failing call on this thread ("" if none). Static storage,
 * valid until the next failing call on the same thread. */
const char* star_last_error(void);

/* Logical pages one sequence needs: ceil((L + round_up(T_max,128)) / page_tokens). */
int star_pages_needed(const star_shape* shape, int32_t* max_pages_out);

/* HOST helper: fill a host int32 array [B][max_pages] with the block-contiguous
 * assignment page_table[s][j] = first_page + s*max_pages + j. */
int star_page_table_fill(const star_shape* shape, int32_t* page_table_host, int32_t max_pages, int32_t first_page);

/* Bytes of scratch the given operation needs (op = STAR_OP_*; for STAR_OP_PHASE2
 * T is the number of query tokens of the call, ignored otherwise).
 * STAR_OP_PHASE1: 0.  STAR_OP_PHASE1_ANCHOR: star_phase1_encode_anchored with anchor
 * position ids, B*(n-1)*Hkv*a*d*2 bytes (the anchor's keys roped at those ids).
 * STAR_OP_PHASE2: RoPE(q) (B*T*Hq*d*2 bytes, rounded up to 256), plus the f32 partials
 * of the chunks when blocks are split to fill the GPU.  STAR_OP_PHASE2_PUSH: the same
 * with the chunk partials always staged (star_phase2_partial_shard_push).
 * STAR_OP_DECODE: the chunk partials of one step. */
int star_workspace_size(const star_shape* shape, int op, int32_t T, size_t* bytes_out);

/* Integer structure of c' ("被增广的上下文"), for checking only.
 * pos_ctx:   device int32 [B][L], position id of each context token (normally t).
 * aug_pos:   device int32 [B][L + (n-1)*a], position ids of c' = [c_1, (a_1 c_2), ...,
 *            (a_1 c_n)] with a_1 the anchor (the first a = shape->anchor tokens of c_1, a = b
 *            by default): block 1 then, per block i>1, the a anchor ids then c_i's ids.
 * block_map: device int32 [B][L][3]: (block t/b, physical page, slot t % page_tokens).
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE (L != n*b), CAPACITY, CUDA. */
int star_build_positions(const star_shape* shape, const star_cache* cache, const int32_t* pos_ctx,
                         int32_t* aug_pos, int32_t* block_map, star_stream_t stream);

/* Append tokens to the cache ("仓库里的真实实现": the last block's owner appends the
 * query and generated tokens' KV; "局部注意力与 KV 丢弃" for the context).
 * k, v: bf16 [B][ntok][Hkv][d]; pos: device int32 [B][ntok] (RoPE positions of K).
 * Writes RoPE(K) and V into cache slots [start, start + ntok) of every sequence.
 * Errors: INVALID_ARG, ALIGNMENT, CAPACITY (start + ntok beyond the page table), CUDA. */
int star_kv_append(const star_shape* shape, const star_cache* cache, const void* k, const void* v,
                   const int32_t* pos, int32_t start, int32_t ntok, star_stream_t stream);

/* Phase 1: anchor-augmented blockwise-local causal attention plus the KV cache
 * ("Phase 1: 被增广的上下文", "局部注意力与 KV 丢弃", "复杂度分析").
 * q: bf16 [B][L][Hq][d]; k, v: bf16 [B][L][Hkv][d]; pos_ctx: device int32 [B][L].
 * Writes out: bf16 [B][L][Hq][d], where row t of block i attends to the anchor
 * keys [0, a) (for i > 1; a = shape->anchor, b by default) and to its own block's keys
 * up to t, each key roped at its own position id.  Writes RoPE(K), V of the L context tokens into cache
 * slots [0, L) (the anchor copies are never written) and zeroes slots
 * [L, L + round_up(T_max,128)).  out also serves as the staging buffer of RoPE(q)
 * during the call (each row is rotated there, then overwritten by its output), so
 * out may be q itself but must not partly overlap q, k or v.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, ALIGNMENT, CAPACITY, CUDA. */
int star_phase1_encode(const star_shape* shape, const star_cache* cache, const void* q, const void* k,
                       const void* v, const int32_t* pos_ctx, void* out, void* ws, size_t ws_bytes,
                       star_stream_t stream);

/* Phase 1 with the anchor's position ids given per block (the anchor variants of
 * "仓库里的真实实现" and the implementers' notes on that page: the anchor's ids may be
 * sampled from the prefix range, or reset to 0, instead of keeping tokens 0..a-1's ids).
 * anchor_pos: device int32 [B][n-1][a]; row i-2 holds the ids of the anchor's a tokens in
 * block i (2 <= i <= n).  NULL: the anchor keeps the ids of tokens 0..a-1 (pos_ctx), exactly
 * star_phase1_encode.  Otherwise the anchor's keys RoPE(k_j, anchor_pos[..][j]) are
 * written into ws (bf16 [B][n-1][Hkv][a][d], star_workspace_size(STAR_OP_PHASE1_ANCHOR))
 * and read from there; the anchor's values are block 1's cached values (V has no
 * position).  The cache contents are the same as star_phase1_encode's.
 * Errors: as star_phase1_encode; CAPACITY if ws_bytes is too small. */
int star_phase1_encode_anchored(const star_shape* shape, const star_cache* cache, const void* q, const void* k,
                                const void* v, const int32_t* pos_ctx, const int32_t* anchor_pos, void* out,
                                void* ws, size_t ws_bytes, star_stream_t stream);

/* Phase 2 per-block partials ("Phase 2: 局部注意力与本地统计量": A_h and s_h per host).
 * q: bf16 [B][T][Hq][d]; k, v: bf16 [B][T][Hkv][d] or both NULL (already appended);
 * q_pos: device int32 [B][T], RoPE positions (normally L + t).
 * If k, v are given they are appended first at cache slots [L, L+T) (tail of the
 * last block).  Query token t (cache index L + t) sees all keys of blocks 1..n-1
 * and, in block n, its b context keys plus tail keys L..L+t.
 * o_part: f32 [n][B][T][Hq][d], normalised local outputs A_i;
 * lse_part: f32 [n][B][T][Hq], log s_i.  T <= T_max.
 * ws: at least star_workspace_size(STAR_OP_PHASE2, T) bytes (never NULL).
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, ALIGNMENT, CAPACITY, CUDA. */
int star_phase2_partial(const star_shape* shape, const star_cache* cache, const void* q, const void* k,
                        const void* v, const int32_t* q_pos, int32_t T, float* o_part, float* lse_part, void* ws,
                        size_t ws_bytes, star_stream_t stream);

/* Exact merge of partials ("组装全局结果"; log-sum-exp form of "数值稳定性").
 * o_part: f32 [n_parts][rows][d]; lse_part: f32 [n_parts][rows].
 * out: bf16 [rows][d] = sum_i exp(LSE_i - LSE) O_i; lse_out: f32 [rows] =
 * log sum_i exp(LSE_i) (may be NULL).  Partials with non-finite LSE are skipped;
 * a row with none gives O = 0, LSE = -inf.  With the layouts of
 * star_phase2_partial, rows = B*T*Hq.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE (d), ALIGNMENT, CUDA. */
int star_lse_merge(int32_t n_parts, int64_t rows, int32_t d, const float* o_part, const float* lse_part, void* out,
                   float* lse_out, star_stream_t stream);

/* One generated token per sequence ("Star Attention: Efficient LLM Inference over
 * Long Sequences", abstract: response tokens attend to all prior cached tokens).
 * q: bf16 [B][1][Hq][d]; k, v: bf16 [B][1][Hkv][d]; pos: device int32 [B].
 * Appends RoPE(k), v at cache slot cur_len, then attends over slots [0, cur_len]
 * (the whole cache including the new token), split into chunks whose (O, LSE)
 * partials are merged exactly.  out: bf16 [B][1][Hq][d]; lse_out: f32 [B][Hq]
 * (may be NULL).  cur_len < L + T_max.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, ALIGNMENT, CAPACITY, CUDA. */
int star_decode_step(const star_shape* shape, const star_cache* cache, const void* q, const void* k, const void* v,
                     const int32_t* pos, int32_t cur_len, void* out, float* lse_out, void* ws, size_t ws_bytes,
                     star_stream_t stream);

/* star_decode_step without a caller workspace.  The Star Attention pages have no
 * counterpart to this call: it exists for callers that cannot call cudaMalloc, such
 * as a serving runtime that reserves all device memory for its own pool at start-up
 * and forbids allocation afterwards, or a plugin that only receives input and
 * output buffers from the application hosting it.  Arguments, layouts and results
 * are those of star_decode_step minus (ws, ws_bytes).
 * Scratch: a 16 MiB device array built into the library (every GPU that loads the
 * library holds it until the process exits).  The first call made on a device
 * looks up that array's device address with cudaGetSymbolAddress, so make that
 * first call before any stream capture (a first call made while `stream` is being
 * captured is refused with STAR_ERR_INVALID_ARG).  All calls share the one array and a call
 * writes every value it later reads, so nothing has to be cleared between calls,
 * but calls whose kernels overlap on the GPU (other streams, other threads) race
 * on it: serialise them.  No device memory is allocated or freed.
 * Errors: those of star_decode_step, plus CAPACITY when the shape's decode partials
 * (star_workspace_size(shape, STAR_OP_DECODE, ...)) exceed 16 MiB. */
int star_decode_step_noalloc(const star_shape* shape, const star_cache* cache, const void* q, const void* k,
                             const void* v, const int32_t* pos, int32_t cur_len, void* out, float* lse_out,
                             star_stream_t stream);

/* Multi-layer context encoding ("仓库里的真实实现": every augmented block [a_1; c_i] runs
 * the whole model forward on its own, and the anchor's part of every layer's KV is
 * dropped).  The caller owns the model: for each layer the library calls `fn` twice,
 * and `fn` enqueues the caller's own kernels (projections, residuals, MLP, ...) on
 * `stream`:
 *   fn(layer, STAR_LAYER_QKV, x, q, k, v, user, stream): q, k, v (pre-RoPE, the
 *       layouts of star_phase1_encode) from the hidden states x;
 *   fn(layer, STAR_LAYER_OUT, o, x, NULL, NULL, user, stream): the next hidden states
 *       into x (in place) from the attention output o = star_phase1_encode(q, k, v).
 * Between the two calls the library runs star_phase1_encode with layer's cache
 * caches[layer].  The anchor is a prefix of block 1 with block 1's position ids, and
 * attention is causal, so at every layer its hidden states, and its keys and values,
 * are block 1's: one pass over the L real tokens per layer gives every block the
 * anchor the pages recompute per host, exactly.  Anchor position ids other than
 * block 1's would break that equality, so this call takes none.
 * x: caller-owned device buffer of the hidden states (its layout is the caller's
 * business; the library only passes it to fn).  q, o: bf16 [B][L][Hq][d]; k, v: bf16
 * [B][L][Hkv][d], caller-owned scratch reused by every layer.  caches: n_layers
 * caches (host array of star_cache), each as for star_phase1_encode.
 * Errors: those of star_phase1_encode; CALLBACK if fn returns non-zero (the call stops
 * there; work already enqueued stays enqueued). */
enum { STAR_LAYER_QKV = 0, STAR_LAYER_OUT = 1 };
typedef int (*star_layer_fn)(int32_t layer, int32_t stage, void* in, void* out0, void* out1, void* out2, void* user,
                             star_stream_t stream);
int star_encode_layers(const star_shape* shape, int32_t n_layers, const star_cache* caches, const int32_t* pos_ctx,
                       void* x, void* q, void* k, void* v, void* o, star_layer_fn fn, void* user,
                       star_stream_t stream);

/* ---------------------------------------------------------------------------
 * Shards: Star Attention across several GPUs, one contiguous block range per GPU.
 * The pages run one host per block ("Star Attention 完全拆解(一)", Phase 1: every host
 * receives the anchor block c_1 with its own block; "仓库里的真实实现": only the host
 * holding the last block appends the query and generated tokens' KV; "通信量:每层每
 * token 一个标量加一个向量": per query token and layer each host contributes one
 * (output, log-sum-exp) pair, which "组装全局结果" merges exactly).  Here a GPU owns
 * blocks [block_begin, block_end) of every sequence; its partials are exchanged (an
 * all-gather or a gather to the GPU that needs the output; the library leaves the
 * transport to the caller's NCCL) and merged with star_lse_merge.
 * The shape is the whole problem's (L = n*b, T_max); sequences must have one length
 * (shape->seq_len NULL).  The cache of a shard holds its own blocks at their cache
 * slots [block_begin*b, block_end*b), plus block 1's first a (anchor) tokens at slots
 * [0, a) when block_begin > 0, plus the tail on the shard with block_end == n; its page
 * table must cover all logical pages those occupy (the rest is never read).
 * ------------------------------------------------------------------------- */
typedef struct star_shard {
  int32_t block_begin; /* first block of the range (0-based) */
  int32_t block_end;   /* one past the last; 0 <= block_begin < block_end <= n */
} star_shard;

/* Phase 1 of a shard's blocks.  q: bf16 [B][R][Hq][d], k, v: bf16 [B][R][Hkv][d] and pos:
 * int32 [B][R] for the range's R = (block_end - block_begin)*b context tokens;
 * out: bf16 [B][R][Hq][d] (may be q; staging as in star_phase1_encode).  k_anchor,
 * v_anchor: bf16 [B][a][Hkv][d] and pos_anchor: int32 [B][a], the anchor's tokens (block
 * 1's first a), required when block_begin > 0 (ignored otherwise).  Writes the range's
 * RoPE(K), V and, when block_begin > 0, the anchor's into the cache; the shard holding
 * the last block also zeroes the tail slots.  Rows equal those of star_phase1_encode.
 * Errors: those of star_phase1_encode; INVALID_ARG for a bad range. */
int star_phase1_encode_shard(const star_shape* shape, const star_cache* cache, const star_shard* shard, const void* q,
                             const void* k, const void* v, const int32_t* pos, const void* k_anchor,
                             const void* v_anchor, const int32_t* pos_anchor, void* out, star_stream_t stream);

/* Phase-2 partials of a shard's blocks: as star_phase2_partial, restricted to blocks
 * [block_begin, block_end).  o_part: f32 [R_b][B][T][Hq][d], lse_part: f32 [R_b][B][T][Hq]
 * with R_b = block_end - block_begin.  k, v (the query's, appended at [L, L+T)) only on the
 * shard holding the last block, whose last partial includes the causal tail; NULL elsewhere.
 * ws: star_workspace_size(STAR_OP_PHASE2, T) bytes.
 * Errors: those of star_phase2_partial; INVALID_ARG for a bad range or k, v off the tail. */
int star_phase2_partial_shard(const star_shape* shape, const star_cache* cache, const star_shard* shard, const void* q,
                              const void* k, const void* v, const int32_t* q_pos, int32_t T, float* o_part,
                              float* lse_part, void* ws, size_t ws_bytes, star_stream_t stream);

/* One decode token's partial over a shard's keys: the range's context keys and, on the
 * shard holding the last block, the tail up to and including the new token (its RoPE(k),
 * v appended at cache slot cur_len there; k, v ignored elsewhere).  q: bf16 [B][1][Hq][d];
 * pos: int32 [B] (the token's position, every shard).  o_part: f32 [B][Hq][d] (normalised
 * local output), lse_part: f32 [B][Hq]; merging every shard's pair with star_lse_merge
 * gives star_decode_step's output.  ws: star_workspace_size(STAR_OP_DECODE) bytes.
 * Errors: those of star_decode_step; INVALID_ARG for a bad range. */
int star_decode_partial_shard(const star_shape* shape, const star_cache* cache, const star_shard* shard, const void* q,
                              const void* k, const void* v, const int32_t* pos, int32_t cur_len, float* o_part,
                              float* lse_part, void* ws, size_t ws_bytes, star_stream_t stream);

/* The exchange over peer memory (NVLink): instead of gathering the partials with a
 * collective library, the kernel that finishes a shard's partials stores them straight
 * into every GPU's exchange buffer, and the merge waits for them there.
 *
 * Each rank allocates ONE exchange buffer of star_exchange_size(world, slots, rows, d)
 * bytes in its own device memory, zero-filled once before its first use (afterwards the
 * calls keep it consistent), maps every other rank's buffer into its process
 * (star_ipc_export / star_ipc_open; peers[w] = rank w's buffer, peers[rank] = its own),
 * and numbers its exchanges 1, 2, 3, ... (epoch), in the same order on every rank.
 * Exchange e uses parity e & 1 of every buffer; a push of epoch e first waits until every
 * rank has merged epoch e - 2 (no barrier).  Every wait is bounded (2 s): a rank that
 * never arrives makes the waiting kernel record STAR_ERR_TIMEOUT (star_device_status) and
 * return.  One buffer serves one kind of exchange (one rows x slots shape). */
typedef struct star_exchange {
  int32_t world;    /* ranks, 1..8 */
  int32_t rank;     /* this rank */
  int32_t slots;    /* partials each rank contributes per exchange (ceil(n / world) for Phase 2, 1 for decode) */
  void* peers[8];   /* device addresses of every rank's exchange buffer as mapped here; 256-byte aligned */
} star_exchange;

/* Bytes of one rank's exchange buffer for exchanges of `slots` partials of `rows` rows of
 * head dim d per rank: a 256-byte header plus 2 x world x (slots*rows*(d+1)*4, each part
 * rounded up to 256). */
int star_exchange_size(int32_t world, int32_t slots, int64_t rows, int32_t d, size_t* bytes_out);

/* star_phase2_partial_shard, with the shard's per-block partials pushed into slot `rank` of
 * every rank's exchange buffer (epoch) instead of written to o_part / lse_part; the slots
 * past the shard's blocks get empty partials (O = 0, LSE = -inf).  rows = B*T*Hq.
 * ws: star_workspace_size(STAR_OP_PHASE2_PUSH, T) bytes.  ex->slots >= the shard's blocks. */
int star_phase2_partial_shard_push(const star_shape* shape, const star_cache* cache, const star_shard* shard,
                                   const void* q, const void* k, const void* v, const int32_t* q_pos, int32_t T,
                                   const star_exchange* ex, uint64_t epoch, void* ws, size_t ws_bytes,
                                   star_stream_t stream);

/* star_decode_partial_shard, with the shard's (O, LSE) pushed into slot `rank` of every
 * rank's exchange buffer (one slot, rows = B*Hq).  ws: star_workspace_size(STAR_OP_DECODE). */
int star_decode_partial_shard_push(const star_shape* shape, const star_cache* cache, const star_shard* shard,
                                   const void* q, const void* k, const void* v, const int32_t* pos, int32_t cur_len,
                                   const star_exchange* ex, uint64_t epoch, void* ws, size_t ws_bytes,
                                   star_stream_t stream);

/* Waits until every rank's partials of `epoch` are in this rank's buffer, merges the
 * world x slots partials of each row ("组装全局结果", log-sum-exp form of "数值稳定性") into
 * out (bf16 [rows][d]) and lse_out (f32 [rows], may be NULL), then tells every rank that
 * this rank's slots of the epoch's parity may be reused. */
int star_exchange_merge(const star_exchange* ex, int64_t rows, int32_t d, uint64_t epoch, void* out, float* lse_out,
                        star_stream_t stream);

/* CUDA IPC for the exchange buffers (host calls): export a device pointer of this process
 * as a 64-byte handle plus its offset in its allocation; open a peer's handle (the pointer
 * is valid in this process, peer access enabled); close it when done. */
int star_ipc_export(const void* ptr, void* handle_out /* 64 bytes */, uint64_t* offset_out);
int star_ipc_open(const void* handle /* 64 bytes */, uint64_t offset, void** ptr_out);
int star_ipc_close(void* ptr, uint64_t offset);

/* Tracing: when both are non-NULL (cudaEvent_t handles created by the caller),
 * every later call on this thread records `start_event` on its stream right
 * before launching its main kernel and `stop_event` right after it (Phase 1 and
 * Phase 2: the tensor-core attention kernel; decode: the split-KV kernel), so the
 * caller can time that kernel with cudaEventElapsedTime.  NULL, NULL turns it off.
 * Errors: INVALID_ARG if exactly one is NULL. */
int star_set_trace_events(void* start_event, void* stop_event);

/* Synchronises `stream`, then reads and clears the device error words that the
 * kernels set when a bounded wait runs out, a page-table entry is out of range, or
 * a merged partial carries a NaN or +inf log-sum-exp.  *status_out receives the raw
 * code (0 = none; 1-3 a wait that ran out, 4 a bad page, 5 a bad partial).  Returns
 * STAR_ERR_TIMEOUT if a wait ran out, STAR_ERR_CAPACITY for a bad page,
 * STAR_ERR_INVALID_ARG for a bad partial, STAR_ERR_CUDA if the stream failed. */
int star_device_status(star_stream_t stream, int32_t* status_out);

/* Failure-detection test hook.  The Star Attention pages have no counterpart to
 * this call: it lets a test watch the kernels' bounded waits give up without
 * faulting or hanging the GPU.  wait_limit_ns: how long any mbarrier wait in the
 * attention and decode kernels may last before the kernel records
 * STAR_ERR_TIMEOUT's code and returns (0 restores the default of 2 s).  flags:
 * STAR_DEBUG_SKIP_FIRST_LOAD makes CTA 0's producer of every later attention and
 * decode launch issue no first K-tile load, so the barrier of that stage never
 * completes, every role's bounded wait runs out, and nothing asynchronous is left
 * in flight (0 = normal operation).  The settings hold for the current device
 * until changed; call it between launches, never while kernels run.
 * Errors: INVALID_ARG (unknown flag), CUDA. */
enum { STAR_DEBUG_SKIP_FIRST_LOAD = 1 };
int star_debug_set(uint64_t wait_limit_ns, int32_t flags);

#ifdef __cplusplus
}
#endif

#endif /* STAR_H_ */
