/*
 * qsa.h — C ABI of the B200 (sm_100a) QSA decode hot path.
 *
 * QSA (Qwen Sparse Attention) decode, as described on the web page
 * "第10回 EVO-X2（Ryzen AI Max+ 395 / 128GB）+ Qwen3.8-Flash-Next用のllama.cpp改造で
 * 長コンテキストのTGを高速化した話" ("Part 10" below), runs in four stages per layer:
 *   1. indexer keys are summarised per 4-token micro-block (mean pool -> RMS norm ->
 *      RoPE at the block position) into a persistent pooled-key cache that is only
 *      extended by newly completed blocks            (Part 10, section COMMON-004);
 *   2. the current indexer query scores every completed block and the top-k blocks
 *      covering indexer_top_k tokens are chosen      (Part 10, sections "QSA indexer",
 *                                                      COMMON-006);
 *   3. their cells plus the open tail block are gathered (at most 2048 + 4 - 1 = 2051)
 *                                                     (Part 10, section COMMON-005);
 *   4. GQA softmax attention runs over those cells only.
 *
 * Conventions shared by every call:
 *  - All data pointers are DEVICE pointers unless stated otherwise. Every buffer is
 *    owned by the caller (e.g. allocated with PyTorch); the library never allocates
 *    device memory and owns only the host-side context.
 *  - Every call that takes a stream is asynchronous on that stream (NULL = legacy
 *    default stream) and returns after HOST-side argument validation only; kernels are
 *    launched with programmatic dependent launch so that consecutive calls on one
 *    stream overlap their launch latency, and all of them are safe to capture in a
 *    CUDA graph. The exceptions synchronise and must stay outside a capture:
 *    qsa_read_layer_state, qsa_n_ctx and qsa_get_device_status.
 *  - A context is not internally locked: use it from one host thread at a time.
 *    Separate contexts are independent.
 *  - The sequence state of each layer (context length n_ctx and number of pooled
 *    blocks n_pooled) lives in DEVICE memory inside the layer's workspace and is
 *    advanced by the kernels themselves, so a captured decode step can be replayed.
 *  - Conditions that depend on that device state (capacity exceeded, a stale pooled
 *    cache, an out-of-range cell or block id) never fault: the kernel skips the
 *    offending work, writes empty outputs and records the first error code in the
 *    layer's device status word, which qsa_read_layer_state() returns.
 *  - f16 means IEEE binary16; f32 means IEEE binary32. Every pointer must be 16-byte
 *    aligned; rows are tightly packed (row-major, innermost index last).
 *  - No call throws across the ABI. A failed call returns a non-zero qsa_status and
 *    stores a message retrievable with qsa_last_error().
 */
#ifndef QSA_H_
#define QSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (cudaStream_t). NULL selects the legacy default stream. */
typedef struct CUstream_st* qsa_stream_t;

typedef enum {
  QSA_OK = 0,
  QSA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad layer id, bad size      */
  QSA_ERR_CAPACITY = 2,      /* more tokens than max_ctx                              */
  QSA_ERR_STATE = 3,         /* layer not bound, or pooled cache behind the context   */
  QSA_ERR_CUDA = 4,          /* a CUDA runtime call failed (message has the detail)   */
  QSA_ERR_UNSUPPORTED = 5,   /* shape outside what the kernels are built for          */
  QSA_ERR_BAD_INDEX = 6,     /* device status only: a block or cell id out of range   */
  QSA_ERR_TIMEOUT = 7        /* device status only: a bounded wait inside a kernel gave
                                up (the kernel skipped its remaining work and returned) */
} qsa_status;

/* Static shape of every layer of one model (Part 10, section "QSA indexer"). */
typedef struct {
  int32_t n_layers;       /* QSA layers held by one context (12 in the pages' model)    */
  int32_t max_ctx;        /* token capacity per layer; a multiple of 4, <= 1,048,576    */
  int32_t d_idx;          /* indexer key width: 64 or 128                               */
  int32_t n_idx_heads;    /* indexer heads H: 1, 2, 4, 8 or 16                          */
  int32_t top_k_tokens;   /* indexer_top_k in tokens: a multiple of 4, <= 4092 (pages: 2048) */
  int32_t n_q_heads;      /* attention query heads Hq                                   */
  int32_t n_kv_heads;     /* attention KV heads Hkv; Hq / Hkv in {1, 2, 4, 8}          */
  int32_t head_dim;       /* attention head dimension D: 64 or 128                      */
  float rope_base;        /* RoPE base (10000)                                          */
  float rms_eps;          /* RMS-norm epsilon inside the square root (1e-6)             */
  /* RoPE of the indexer keys and query (Part 10, section "QSA indexer": RoPE at the block
   * position). The pages fix neither the pairing, the rotary width nor the position scale;
   * zero-initialised fields give the defaults below. */
  int32_t rope_dims;        /* rotary dims R: even, 2..d_idx; the rest pass through. 0 = d_idx */
  int32_t rope_interleaved; /* 0: NeoX pairs (i, i+R/2); 1: GPT-J pairs (2i, 2i+1). Pair i
                               turns by pos * rope_base^(-2i/R)                          */
  int32_t rope_pos_stride;  /* block b sits at position stride*b + offset and the query at
                               floor(stride*(n-1)/4): 4 = token positions (block = its first
                               token, query = token n-1), 1 = block indices. 1..16; 0 = 4 */
  int32_t rope_pos_offset;  /* 0..1,048,576 (0)                                          */
  /* Storage of the attention K/V cache (the Qwen3.8-Flash-Next parameter-tuning post on
   * EVO-X2, section "KV cacheをQ8_0にしてみる", tried an 8-bit K/V cache).
   * QSA_KV_F16 (0): f16 rows. QSA_KV_FP8 (1): e4m3 codes with one f32 scale per
   * (token, KV head) row, scale = amax/448, code = e4m3(x * 448/amax) rounded to
   * nearest-even and saturated (an all-zero row: scale 1, zero codes); attention reads
   * code * scale. The indexer caches stay f16 either way. */
  int32_t kv_format;
  /* How the indexer scan computes the dots q~_h . p_b (the scores are the same up to f32
   * rounding; zero gives the default). QSA_SCAN_TENSOR (0): the 5th-generation tensor
   * cores (tcgen05), the query split into f16 high and scaled low parts so it keeps ~22
   * significant bits. QSA_SCAN_CUDA_CORES (1): the CUDA cores, an f32 query and packed
   * f32 FMAs with warp-shuffle reductions; single-query scans only (the multi-query calls
   * use the tensor cores), and a decode step with it takes four launches. */
  int32_t scan_kind;
  /* Storage of the pooled-key cache (the other half of the 8-bit option the tuning post's
   * section "KV cacheをQ8_0にしてみる" tried). QSA_POOLED_F16 (0): f16 summaries.
   * QSA_POOLED_FP8 (1): each f16 summary stored as d_idx e4m3 codes and one f32 scale per
   * row (pooled_scales), by the QSA_KV_FP8 rule; the indexer scores code * scale, on the
   * tensor cores with 8-bit operands (d_idx 128, QSA_SCAN_TENSOR and single-query scans
   * only: otherwise QSA_ERR_UNSUPPORTED). The scan then reads half the bytes. */
  int32_t pooled_format;
  /* When a call may read its inputs (token rows, queries, head weights).
   * QSA_INPUTS_ORDERED (0): only after the previous work on the stream has completed.
   * QSA_INPUTS_EARLY (1): the caller guarantees that every input of a call is complete in
   * device memory before the call's first kernel can start: written by copies or by
   * kernels that finish first, never by a kernel on the same stream that lets its
   * dependents start early (programmatic dependent launch). The indexer scan then loads
   * and splits the query while the previous kernel still runs. Results are identical. */
  int32_t early_inputs;
} qsa_config;

enum { QSA_KV_F16 = 0, QSA_KV_FP8 = 1 };
enum { QSA_SCAN_TENSOR = 0, QSA_SCAN_CUDA_CORES = 1 };
enum { QSA_POOLED_F16 = 0, QSA_POOLED_FP8 = 1 };
enum { QSA_INPUTS_ORDERED = 0, QSA_INPUTS_EARLY = 1 };

/* Caller-owned device buffers of one layer. Sizes come from qsa_buffer_bytes(). */
typedef struct {
  void* k_cache;          /* [max_ctx][n_kv_heads][head_dim] f16 (e4m3 bytes with
                             QSA_KV_FP8), token-major                                   */
  void* v_cache;          /* same layout as k_cache                                     */
  void* idx_cache;        /* [max_ctx][d_idx] f16: raw per-token indexer keys           */
  void* pooled_cache;     /* [max_ctx/4][d_idx] f16: pooled summaries p_b (e4m3 bytes
                             with QSA_POOLED_FP8)                                        */
  const float* rms_gain;  /* [d_idx] f32 RMS-norm gain, or NULL for unit gain           */
  void* workspace;        /* device state + scratch; QSA_BUF_WORKSPACE bytes            */
  void* kv_scales;        /* QSA_KV_FP8 only: [max_ctx][n_kv_heads][2] f32, the K and V
                             scales of each row; NULL with QSA_KV_F16                   */
  void* pooled_scales;    /* QSA_POOLED_FP8 only: [max_ctx/4] f32, the scale of each
                             pooled row (pooled_cache then holds e4m3 codes); NULL otherwise */
} qsa_layer_buffers;

enum {
  QSA_BUF_KV = 0,         /* bytes of k_cache (v_cache has the same size) */
  QSA_BUF_IDX = 1,        /* bytes of idx_cache                           */
  QSA_BUF_POOLED = 2,     /* bytes of pooled_cache                        */
  QSA_BUF_WORKSPACE = 3,  /* bytes of workspace                           */
  QSA_BUF_MAX_CELLS = 4,  /* not bytes: max cells per step = 4*(top_k_tokens/4) + 3 */
  QSA_BUF_SCORE_STRIDE = 5, /* not bytes: floats per row of a multi-query score table
                               (max_ctx/4 rounded up to a multiple of 64) */
  QSA_BUF_KV_SCALES = 6,  /* bytes of kv_scales (0 with QSA_KV_F16)      */
  QSA_BUF_POOLED_SCALES = 7 /* bytes of pooled_scales (0 with QSA_POOLED_F16) */
};

typedef struct qsa_ctx qsa_ctx;

/* Size in bytes of one of a layer's buffers (see QSA_BUF_*); 0 if cfg is invalid. */
size_t qsa_buffer_bytes(const qsa_config* cfg, int32_t which);

/* Validate cfg and create a host context bound to the CURRENT CUDA device.
 * Returns QSA_ERR_UNSUPPORTED for shapes the kernels are not built for. */
qsa_status qsa_create(const qsa_config* cfg, qsa_ctx** out);

/* Free the host context. Does not touch any device buffer. NULL is a no-op. */
void qsa_destroy(qsa_ctx* ctx);

/* Message of the last failed call on ctx (host string owned by ctx), "" if none. */
const char* qsa_last_error(const qsa_ctx* ctx);

/* Attach a layer's buffers and reset its device state to an empty sequence
 * (n_ctx = n_pooled = 0, status = 0), asynchronously on `stream`. Also encodes the
 * TMA descriptor of the pooled cache. May be called again to rebind. */
qsa_status qsa_bind_layer(qsa_ctx* ctx, int32_t layer, const qsa_layer_buffers* buf,
                          qsa_stream_t stream);

/* State load (Part 10, section COMMON-004: a cache that can no longer be trusted after a
 * state load is invalidated and rebuilt when next needed). Sets the device state to
 * n_ctx tokens of which the first n_pooled blocks already hold valid summaries; the
 * caller has written the K/V/indexer caches (and pooled rows < n_pooled). Requires
 * 0 <= n_pooled <= n_ctx/4 and n_ctx <= max_ctx. Clears the status word. */
qsa_status qsa_restore_layer(qsa_ctx* ctx, int32_t layer, int32_t n_ctx, int32_t n_pooled,
                             qsa_stream_t stream);

/* Synchronise `stream` and read the layer's device state. Any output pointer may be
 * NULL. If clear != 0 the status word is reset to 0 afterwards. */
qsa_status qsa_read_layer_state(qsa_ctx* ctx, int32_t layer, int32_t* n_ctx,
                                int32_t* n_pooled, int32_t* device_status, int32_t clear,
                                qsa_stream_t stream);

/* Append one token at position n_ctx: k, v [n_kv_heads][head_dim] f16 and the raw
 * indexer key idx_key [d_idx] f16 (Part 10, section COMMON-004: the raw indexer K cache
 * is the source of pooling). Device status QSA_ERR_CAPACITY (and no write) if the
 * layer is full. */
qsa_status qsa_append_token(qsa_ctx* ctx, int32_t layer, const void* k, const void* v,
                            const void* idx_key, qsa_stream_t stream);

/* Append n >= 1 tokens (prefill): k, v [n][n_kv_heads][head_dim] f16,
 * idx_key [n][d_idx] f16. All-or-nothing: nothing is written if they do not fit. */
qsa_status qsa_append_tokens(qsa_ctx* ctx, int32_t layer, int32_t n, const void* k,
                             const void* v, const void* idx_key, qsa_stream_t stream);

/* Incremental pooled-key cache update (Part 10, section COMMON-004): computes p_b for
 * exactly the blocks b in [n_pooled, n_ctx/4) — mean of the 4 raw indexer keys,
 * RMS norm (eps, gain), NeoX RoPE at position 4b, stored as f16 — and sets
 * n_pooled = n_ctx/4. In decode this is one block every 4th token, else nothing. */
qsa_status qsa_update_pooled_cache(qsa_ctx* ctx, int32_t layer, qsa_stream_t stream);

/* Decode form of the two calls above in one launch (Part 10, section COMMON-004: in
 * decode only the block the new token completes is pooled): appends one token like
 * qsa_append_token, then pools every block in [n_pooled, (n_ctx+1)/4) like
 * qsa_update_pooled_cache — one block every 4th token, usually none. The result is
 * bit-identical to the two calls. Device status QSA_ERR_CAPACITY (and no write) if the
 * layer is full. */
qsa_status qsa_decode_append(qsa_ctx* ctx, int32_t layer, const void* k, const void* v,
                             const void* idx_key, qsa_stream_t stream);

/* Sequence edit / state load: summaries from block `from_block` on are no longer
 * trusted; sets n_pooled = min(n_pooled, from_block). The next update rebuilds them. */
qsa_status qsa_invalidate_pooled_cache(qsa_ctx* ctx, int32_t layer, int32_t from_block,
                                       qsa_stream_t stream);

/* Indexer scan + block-domain top-k (Part 10, sections "QSA indexer" and COMMON-006).
 *   q_idx  [n_idx_heads][d_idx] f16: the current token's indexer query, NOT yet
 *          rotated; the library applies RoPE at position n_ctx-1.
 *   w      [n_idx_heads] f32: per-head weights.
 *   score_b = sum_h w_h * max(0, RoPE(q_h, n_ctx-1) . p_b) / sqrt(d_idx)
 *   for every completed block b < n_ctx/4, accumulated in f32.
 * Outputs: sel_blocks [top_k_tokens/4] i32 — the min(K, B) highest-scoring blocks,
 * ties to the lower block index, in ascending order; n_sel — a device i32 scalar
 * with their count; scores [max_ctx/4] f32 (optional, may be NULL) — every score.
 * Requires the pooled cache to be current (n_pooled == n_ctx/4); otherwise device
 * status QSA_ERR_STATE and n_sel = 0. */
qsa_status qsa_index_topk(qsa_ctx* ctx, int32_t layer, const void* q_idx, const float* w,
                          int32_t* sel_blocks, int32_t* n_sel, float* scores,
                          qsa_stream_t stream);

/* The two halves of qsa_index_topk, for callers that want the scores alone or want to
 * select from scores they computed. qsa_index_scores writes scores [n_ctx/4] f32 (same
 * definition and requirements as above); qsa_select_topk selects from the first n_ctx/4
 * entries of scores with the same rule and outputs (NaN ranks lowest; -0 equals +0).
 * Both take a scores buffer of max_ctx/4 f32: qsa_select_topk may read all of it (the
 * entries past n_ctx/4 are ignored). */
qsa_status qsa_index_scores(qsa_ctx* ctx, int32_t layer, const void* q_idx, const float* w,
                            float* scores, qsa_stream_t stream);
qsa_status qsa_select_topk(qsa_ctx* ctx, int32_t layer, const float* scores, int32_t* sel_blocks,
                           int32_t* n_sel, qsa_stream_t stream);

/* Selected K/V gather (Part 10, section COMMON-005). Expands the selected blocks into
 * their cells 4b..4b+3 and appends the open tail block [4*(n_ctx/4), n_ctx):
 *   cells [4*(top_k_tokens/4)+3] i32 (ascending when sel_blocks is ascending),
 *   n_cells device i32 scalar = 4*n_sel + n_ctx mod 4.
 * If k_compact / v_compact are non-NULL, also copies the selected rows into them:
 * [max_cells][n_kv_heads][head_dim] f16 each (the literal compact K/V; f16 caches only,
 * QSA_ERR_UNSUPPORTED with QSA_KV_FP8). Block ids out
 * of range are reported as device status QSA_ERR_BAD_INDEX and their cells written as
 * -1, which qsa_sparse_attend skips. */
qsa_status qsa_gather_kv(qsa_ctx* ctx, int32_t layer, const int32_t* sel_blocks,
                         const int32_t* n_sel, int32_t* cells, int32_t* n_cells,
                         void* k_compact, void* v_compact, qsa_stream_t stream);

/* GQA attention over the selected cells, reading K/V rows straight from the cache
 * (the gather fused into a split-KV flash-decode; Part 10, section COMMON-005).
 *   q     [n_q_heads][head_dim] f16, already position-encoded by the model;
 *   cells [n_cells] i32 device ids in [0, n_ctx); n_cells device i32 scalar
 *         (<= max cells); out [n_q_heads][head_dim] f32.
 *   out_i = sum_c softmax_c(q_i . K[c][g] / sqrt(D)) V[c][g], g = i / (Hq/Hkv),
 *   with f32 softmax and accumulation. An empty cell set gives out = 0; ids out of
 *   range are skipped and reported as device status QSA_ERR_BAD_INDEX. */
qsa_status qsa_sparse_attend(qsa_ctx* ctx, int32_t layer, const void* q, const int32_t* cells,
                             const int32_t* n_cells, float* out, qsa_stream_t stream);

/* qsa_gather_kv's cell expansion fused into qsa_sparse_attend (Part 10, sections
 * COMMON-005 and COMMON-006: expand only the chosen blocks into cells, add the tail
 * index, attend over those rows). Takes the selection straight from qsa_index_topk /
 * qsa_select_topk: sel_blocks [n_sel] i32 ascending block ids (< n_ctx/4), n_sel a
 * device i32 scalar (<= top_k_tokens/4). The cell set is {4b..4b+3 : b in sel} plus
 * [4*(n_ctx/4), n_ctx), exactly as qsa_gather_kv writes it; output as qsa_sparse_attend.
 * Out-of-range block ids are skipped and reported as device status QSA_ERR_BAD_INDEX. */
qsa_status qsa_sparse_attend_selected(qsa_ctx* ctx, int32_t layer, const void* q,
                                      const int32_t* sel_blocks, const int32_t* n_sel, float* out,
                                      qsa_stream_t stream);

/* ---- Multi-query step: speculative / multi-token verification ----
 * Part 10 (section COMMON-004) requires that speculative decoding's dirty writes never
 * corrupt the cached pooled range. A verification step appends T drafted tokens
 * (qsa_append_tokens, then qsa_update_pooled_cache), scores, selects and attends for
 * all T queries at once, then drops the rejected tokens with qsa_rollback. Query u
 * (u < T) belongs to token n_ctx - T + u and sees exactly what a single-token step at
 * that token would: the blocks completed within its first n_ctx - T + u + 1 tokens and
 * its own open tail. T ranges over 1..4. */
#define QSA_MAX_QUERIES 4

/* qsa_index_topk for T queries in one pass over the pooled cache (one launch of the
 * scan, one of the selection):
 *   q_idx [T][n_idx_heads][d_idx] f16 (un-rotated; query u is rotated at its own
 *         token's position), w [T][n_idx_heads] f32;
 *   sel_blocks [T][top_k_tokens/4] i32 (row u ascending), n_sel [T] device i32;
 *   scores: NULL (the layer workspace holds them) or [T][S] f32 with S =
 *         qsa_buffer_bytes(cfg, QSA_BUF_SCORE_STRIDE); row u is meaningful for blocks
 *         < (n_ctx - T + u + 1)/4, later entries are not part of the result.
 * Requires the pooled cache to be current for the whole context (n_pooled == n_ctx/4)
 * and n_ctx >= T - 1; otherwise device status QSA_ERR_STATE and n_sel = 0. */
qsa_status qsa_index_topk_multi(qsa_ctx* ctx, int32_t layer, int32_t n_queries, const void* q_idx,
                                const float* w, int32_t* sel_blocks, int32_t* n_sel, float* scores,
                                qsa_stream_t stream);

/* qsa_sparse_attend_selected for T queries in one launch: q [T][n_q_heads][head_dim]
 * f16, sel_blocks [T][top_k_tokens/4] and n_sel [T] as qsa_index_topk_multi writes
 * them, out [T][n_q_heads][head_dim] f32. Query u attends over its selected blocks and
 * the tail [4*(n_u/4), n_u), n_u = n_ctx - T + u + 1. */
qsa_status qsa_sparse_attend_selected_multi(qsa_ctx* ctx, int32_t layer, int32_t n_queries, const void* q,
                                            const int32_t* sel_blocks, const int32_t* n_sel, float* out,
                                            qsa_stream_t stream);

/* Drop the tokens at positions >= n_keep (the rejected drafts): n_ctx = min(n_ctx,
 * n_keep) and n_pooled = min(n_pooled, n_ctx/4) on the device, so summaries of blocks
 * that rejected tokens completed are recomputed by the next pooled update (or
 * qsa_decode_append). The cache rows past n_keep are left as they are and overwritten
 * by later appends. n_keep >= 0; a larger n_keep than n_ctx changes nothing. */
qsa_status qsa_rollback(qsa_ctx* ctx, int32_t layer, int32_t n_keep, qsa_stream_t stream);

/* ---- Conveniences ---- */

/* Same as qsa_buffer_bytes (the sizing helper under its other name). */
size_t qsa_layer_bytes(const qsa_config* cfg, int32_t which);

/* Tokens in the layer's caches. The sequence state lives on the device (so that captured
 * steps replay without the host), so this synchronises the device and reads it. Returns
 * -1 if ctx or layer is invalid or the read fails. */
int32_t qsa_n_ctx(const qsa_ctx* ctx, int32_t layer);

/* Synchronise the device and report device-side errors: *status_out = the first non-zero
 * status word over the bound layers in layer order (QSA_OK if none). The status words are
 * left as they are (qsa_read_layer_state clears one). Returns QSA_ERR_CUDA if the device
 * reports a CUDA error. */
qsa_status qsa_get_device_status(qsa_ctx* ctx, int32_t* status_out);

/* One decode step of one layer, the whole hot path on `stream`: the append of the
 * token (k, v, idx_key) with the incremental pooled update, the indexer scan of q_idx / w
 * into the layer workspace, the block top-k into sel_blocks / n_sel, and the sparse
 * attention of q over the selection into out. Arguments as in qsa_decode_append,
 * qsa_index_topk and qsa_sparse_attend_selected; the results are bit-identical to making
 * those three calls one by one.
 * Launches: when the pooled cache is current up to the previous token (the library knows
 * that from the calls made on the layer: after qsa_update_pooled_cache, qsa_decode_append,
 * qsa_decode_step or qsa_rollback, not after qsa_append_token(s), qsa_restore_layer with
 * blocks left to pool or qsa_invalidate_pooled_cache), three: the scan kernel itself
 * appends the token and pools the block the token completes (Part 10, section
 * "incremental pooled-key cache（COMMON-004）": only the new block is computed), then the
 * selection, then the attention. Otherwise four: a separate append that pools every
 * waiting block first. If the device state disagrees (the pooled cache is behind), the
 * three-launch form appends nothing and reports QSA_ERR_STATE in the device status. */
qsa_status qsa_decode_step(qsa_ctx* ctx, int32_t layer, const void* k, const void* v, const void* idx_key,
                           const void* q_idx, const float* w, const void* q, int32_t* sel_blocks,
                           int32_t* n_sel, float* out, qsa_stream_t stream);

/* ---- Context-parallel decode step (one layer sharded over devices) ----
 * Part 10 (section "QSAとQSA indexerについて") handles long context by sparsity: the
 * attended set stays at most 4K + 3 cells whatever the context length. For a context
 * beyond one device, each device holds a contiguous, block-aligned shard of the layer as
 * its own layer: global blocks [block_base, block_base + its n_ctx/4) and, on the last
 * shard only, the open tail. Its config has rope_pos_offset = rope_pos_stride *
 * block_base (plus the unsharded layer's own offset), so its blocks are pooled at their
 * global positions; appends and pooled updates are the ordinary calls. One step:
 *   1. every shard: qsa_cp_index_candidates (its local top-K as fixed-size slots);
 *   2. the slots of all shards, shard by shard, gathered on every device (for instance an
 *      all-gather of K floats and K ints per shard), then qsa_cp_select: the global
 *      top-K, identical on every device;
 *   3. every shard: qsa_cp_attend_partial over its part of the global selection;
 *   4. the partials (out, lse) gathered, then qsa_cp_merge.
 * The result equals the single-device step on the whole context: every block of the
 * global top-K is in its own shard's local top-K, and candidates listed shard by shard in
 * block order keep ties going to the lower block. The exchange itself is the caller's
 * (NCCL or any collective); these calls only compute. */

/* The shard's indexer scan with the query at global position n_global - 1 (rotated there,
 * as the single-device scan rotates it at n_ctx - 1), then its local top-K:
 *   cand_scores [top_k_tokens/4] f32, cand_blocks [top_k_tokens/4] i32: the selected
 *   blocks' scores and GLOBAL ids (local id + block_base) in ascending block order; the
 *   slots past the count hold -inf and -1; n_cand: a device i32, the count.
 * Uses the layer workspace's score buffer. Requires the shard's pooled cache to be
 * current (else QSA_ERR_STATE in the device status and n_cand = 0, all slots empty). */
qsa_status qsa_cp_index_candidates(qsa_ctx* ctx, int32_t layer, const void* q_idx, const float* w, int32_t n_global,
                                   int32_t block_base, float* cand_scores, int32_t* cand_blocks, int32_t* n_cand,
                                   qsa_stream_t stream);

/* The global top-K of every shard's slots: cand_scores [n_shards][k_blocks] f32 and
 * cand_blocks [n_shards][k_blocks] i32 as qsa_cp_index_candidates writes them, shard by
 * shard in block order. Rule of the single-device selection: the k_blocks largest scores,
 * ties to the lower block, ascending; fewer candidates than k_blocks: all of them.
 * Writes sel_blocks [k_blocks] (global ids) and n_sel (device i32). Needs no context:
 * n_shards * k_blocks <= 8192 (QSA_ERR_UNSUPPORTED beyond), k_blocks <= 1024. */
qsa_status qsa_cp_select(const float* cand_scores, const int32_t* cand_blocks, int32_t n_shards, int32_t k_blocks,
                         int32_t* sel_blocks, int32_t* n_sel, qsa_stream_t stream);

/* The shard's attention partial: over the blocks of the global selection (sel_blocks,
 * n_sel from qsa_cp_select, so in ascending order; other orders are not supported) that
 * fall in [block_base, block_base + n_ctx/4), plus the
 * shard's own open tail (the last shard's), like qsa_sparse_attend_selected:
 *   out [n_q_heads][head_dim] f32: the normalised output over those cells;
 *   lse [n_q_heads] f32: log sum_c exp(q_i . K[c] / sqrt(head_dim)); -inf and out = 0 when
 *   the shard has no cell. Uses the layer workspace. */
qsa_status qsa_cp_attend_partial(qsa_ctx* ctx, int32_t layer, const void* q, const int32_t* sel_blocks,
                                 const int32_t* n_sel, int32_t block_base, float* out, float* lse,
                                 qsa_stream_t stream);

/* The exact merge of the shards' partials: o_parts [n_shards][n_q_heads][head_dim] f32,
 * lse_parts [n_shards][n_q_heads] f32 -> out [n_q_heads][head_dim] f32,
 * out = sum_r exp(lse_r - L) o_r / sum_r exp(lse_r - L), L = max_r lse_r (shards with lse
 * -inf count 0; all of them: out = 0). Needs no context. */
qsa_status qsa_cp_merge(const float* o_parts, const float* lse_parts, int32_t n_shards, int32_t n_q_heads,
                        int32_t head_dim, float* out, qsa_stream_t stream);

/* Size of the fixed scratch array behind qsa_sparse_attend_noalloc (1 MiB). */
#define QSA_NOALLOC_SCRATCH_BYTES (1u << 20)

/* qsa_sparse_attend without a context, a workspace or any other scratch from the caller.
 * The pages have no counterpart: it exists for callers that cannot call cudaMalloc —
 * for instance a plugin inside a serving runtime that reserves all device memory in
 * its own arena and forbids further allocations, or a process under a hard
 * device-memory cap — and so cannot provide the layer workspace that holds the
 * split-KV partials. The caller passes only inputs and the output:
 *   q [n_q_heads][head_dim] f16; k_cache, v_cache [>= n_ctx][n_kv_heads][head_dim] f16;
 *   cells [n_cells] i32 device ids (ids outside [0, n_ctx) are skipped); n_cells a device
 *   i32 scalar, at most 4*(top_k_tokens/4)+3; out [n_q_heads][head_dim] f32.
 * The result is the same as qsa_sparse_attend's for the same inputs and shapes.
 * Scratch: one array of QSA_NOALLOC_SCRATCH_BYTES compiled into the library; every GPU
 * that loads the library holds it until the process exits. The first call on a device
 * looks up the array's device address (make that first call before any stream capture);
 * later calls reuse it while the device keeps the same CUDA context, and look it up again
 * after the context was replaced (a device reset or a primary-context teardown). With no
 * valid cells the output rows are zero; a negative *n_cells counts as zero.
 * Every call shares the array and overwrites what the previous call left there, so
 * calls whose kernels overlap on the GPU (on different streams, or from several host
 * threads) race and must be serialised by the caller. Nothing here allocates: no
 * cudaMalloc, cudaFree or allocating library routine is called.
 * Returns QSA_ERR_INVALID_ARG for null or misaligned pointers or n_ctx < 0,
 * QSA_ERR_UNSUPPORTED for shapes the kernels are not built for (head_dim 64/128,
 * n_q_heads/n_kv_heads in {1,2,4,8}, top_k_tokens a positive multiple of 4),
 * QSA_ERR_CAPACITY if the partials of these shapes would not fit in the array, and
 * QSA_ERR_CUDA if a launch fails. Device-side problems are not reported. */
qsa_status qsa_sparse_attend_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                     int32_t n_ctx, const int32_t* cells, const int32_t* n_cells,
                                     float* out, int32_t n_q_heads, int32_t n_kv_heads,
                                     int32_t head_dim, int32_t top_k_tokens, qsa_stream_t stream);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* QSA_H_ */
