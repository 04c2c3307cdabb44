// Internal declarations shared by the library's translation units: the device-side
// sequence state, the workspace layout and the kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/qsa.h"

namespace qsa {

constexpr int kBlock = 4;             // tokens per micro-block (compression ratio 4)
constexpr int kTopkCluster = 16;      // CTAs in the top-k cluster
constexpr int kTopkThreads = 512;
constexpr int kTopkMaxPerCta = kTopkThreads * 32;  // keys held in registers per top-k CTA
constexpr int kTopkMaxK = kTopkThreads * 32 / kTopkCluster;  // largest top_k_tokens / 4 (1024)
constexpr int kMaxQueries = 4;        // queries verified together by the multi-query calls
constexpr int kAttnWarps = 8;         // warps per attention CTA
constexpr int kAttnMaxCells = 64;     // cells per attention CTA (split size cap)
constexpr int kHistBits = 11;         // score-key prefix bits the scan histograms for the selection

// Device-resident sequence state of one layer; lives at the start of the workspace.
struct DevState {
  int32_t n_ctx;          // tokens in the caches
  int32_t n_pooled;       // completed blocks whose summaries are valid
  int32_t status;         // first device-side error (qsa_status), 0 if none
  uint32_t ticket_append; // last-CTA tickets of multi-CTA kernels (reset by the last CTA)
  uint32_t ticket_pool;
  int32_t reserved[59];
};
static_assert(sizeof(DevState) == 256, "DevState must stay 256 bytes");

// Timeline build only (-DQSA_TIMELINE): right after a layer's DevState in its workspace,
// [kernel][point][min, max] of the low 32 bits of %globaltimer (ns) that the CTAs of the
// step's kernels reached at each probe point (kernels: scan, top-k, attention, and detail
// rows of each).
constexpr int kTimelineKernels = 10, kTimelinePoints = 5;
constexpr size_t kTimelineOffset = sizeof(DevState);
constexpr size_t kTimelineBytes = 512;
static_assert(kTimelineKernels * kTimelinePoints * 2 * 4 <= kTimelineBytes, "timeline region");

// Byte offsets inside a layer's workspace (all 256-byte aligned).
struct WorkspaceLayout {
  size_t state, hist, cp, scores, part_o, part_ml, total;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Attention split: each CTA of the split-KV kernel takes `cells_per_cta` cells of one
// KV head; `n_splits` CTAs per KV head cover the largest cell set.
struct AttnSplit {
  int cells_per_cta;
  int n_splits;
};

inline int max_cells_of(const qsa_config& c) { return kBlock * (c.top_k_tokens / kBlock) + kBlock - 1; }

inline AttnSplit attn_split(const qsa_config& c, int n_sms) {
  int max_cells = max_cells_of(c);
  int per_head = n_sms / c.n_kv_heads;
  if (per_head < 1) per_head = 1;
  int l = (max_cells + per_head - 1) / per_head;
  l = (l + 7) / 8 * 8;
  if (l < 8) l = 8;
  if (l > kAttnMaxCells) l = kAttnMaxCells;
  return AttnSplit{l, (max_cells + l - 1) / l};
}

// Row stride (floats) of a multi-query score table: one row per query, 256-byte aligned.
inline int score_stride_of(const qsa_config& c) { return (c.max_ctx / kBlock + 63) / 64 * 64; }

inline WorkspaceLayout workspace_layout(const qsa_config& c, int n_splits) {
  WorkspaceLayout w{};
  size_t off = 0;
  w.state = off;
  off += align256(sizeof(DevState));
  off += kTimelineBytes;  // the timeline build's probe record (kTimelineOffset)
  w.hist = off;  // score-key prefix histograms of the last scan, one per query (zero between selections)
  off += align256(size_t(kMaxQueries) * (1 << kHistBits) * sizeof(uint32_t));
  w.cp = off;    // a context-parallel shard's part of the global selection: count, then ids
  off += align256(size_t(16 + kTopkMaxK) * sizeof(int32_t));
  w.scores = off;  // kMaxQueries rows of score_stride_of(c) floats
  off += align256(size_t(kMaxQueries) * score_stride_of(c) * sizeof(float));
  w.part_o = off;
  off += align256(size_t(n_splits) * c.n_q_heads * c.head_dim * sizeof(float));
  w.part_ml = off;
  off += align256(size_t(n_splits) * c.n_q_heads * 2 * sizeof(float));
  w.total = off;
  return w;
}

// Everything a launcher needs about one bound layer.
struct LayerView {
  qsa_config cfg;
  void* k_cache;
  void* v_cache;
  void* idx_cache;
  void* pooled_cache;
  const float* rms_gain;
  float* kv_scales;       // [max_ctx][n_kv_heads][2] f32 with QSA_KV_FP8, else null
  float* pooled_scales;   // [max_ctx/4] f32 with QSA_POOLED_FP8, else null
  DevState* state;
  float* scores;          // workspace scores
  uint32_t* hist;         // workspace score-key prefix histogram
  int32_t* cp_count;      // workspace: a context-parallel shard's selected-block count
  int32_t* cp_sel;        //            and its local block ids
  float* part_o;
  float* part_ml;
  AttnSplit split;
  int n_sms;
  int attn_cluster;        // CTAs per KV head in the attention cluster (16 or 8)
  int attn_cells_per_cta;  // cells each of them stages
  CUtensorMap pooled_tile_map;  // TMA descriptors of pooled_cache (encoded at bind time):
  CUtensorMap pooled_box_map;   // 128-row boxes for whole tiles, 16-row boxes for ragged ones
};

// ---- launchers (return the launch's cudaError_t) ----
cudaError_t init_kernel_attributes();  // once per context creation, outside any capture
cudaError_t init_scan_attributes();
cudaError_t encode_pooled_map(const qsa_config& c, void* pooled, int box_rows, CUtensorMap* out);
cudaError_t launch_set_state(const LayerView& L, int n_ctx, int n_pooled, int mode, cudaStream_t s);
cudaError_t launch_append(const LayerView& L, int n, const void* k, const void* v,
                          const void* idx, int grid_hint, cudaStream_t s);
cudaError_t launch_pool_update(const LayerView& L, int grid_hint, cudaStream_t s);
cudaError_t launch_decode_append(const LayerView& L, const void* k, const void* v, const void* idx, cudaStream_t s);
// The index/top-k/attention launchers take n_queries T >= 1: query t (t < T) belongs to
// token n_ctx - T + t and sees only the first n_ctx - T + t + 1 tokens. Per-query inputs
// and outputs are consecutive rows (scores: rows of score_stride floats).
// With `hist` (single query only) the scan also fills the score-key prefix histogram and
// the selection starts from it (and clears it for the next scan).
// q_n > 0 (single query): the query belongs to token q_n - 1 of a longer sequence (a
// context-parallel shard's scan), else to token n_ctx - 1.
cudaError_t launch_index_scan(const LayerView& L, const void* q_idx, const float* w,
                              float* scores, cudaStream_t s, int n_queries = 1, int score_stride = 0,
                              uint32_t* hist = nullptr, int q_n = 0);
// With sel_scores (single query), the selection also writes each selected block's score,
// adds block_base to the written ids and pads positions past n_sel with -inf / -1 (the
// fixed-size candidate slots of a context-parallel shard). after_fused_scan: the scan
// before it was the decode step's (launch_decode_scan), which appended the token without
// advancing the state; the selection counts that token and advances the state.
cudaError_t launch_topk(const LayerView& L, const float* scores, int32_t* sel, int32_t* n_sel,
                        cudaStream_t s, int n_queries = 1, int score_stride = 0, uint32_t* hist = nullptr,
                        float* sel_scores = nullptr, int block_base = 0, bool after_fused_scan = false);
// The same scan on the CUDA cores (scan_kind = QSA_SCAN_CUDA_CORES; single query).
cudaError_t init_scan_cc_attributes();
cudaError_t launch_index_scan_cc(const LayerView& L, const void* q_idx, const float* w, float* scores,
                                 uint32_t* hist, cudaStream_t s, int q_n = 0);
// Decode step's first launch: append the token at n_ctx (pooling the block it completes)
// and scan, filling `hist`. Needs the pooled cache current up to the token before.
cudaError_t launch_decode_scan(const LayerView& L, const void* k, const void* v, const void* idx,
                               const void* q_idx, const float* w, float* scores, uint32_t* hist, cudaStream_t s);
cudaError_t launch_gather(const LayerView& L, const int32_t* sel, const int32_t* n_sel,
                          int32_t* cells, int32_t* n_cells, void* k_compact, void* v_compact,
                          cudaStream_t s);
cudaError_t launch_attend(const LayerView& L, const void* q, const int32_t* cells,
                          const int32_t* n_cells, float* out, cudaStream_t s);
// With lse (single query): also the log-sum-exp of each head's scaled logits over its cells.
// warm: the kernel launches well before its inputs are ready (the decode step, behind the
// selection) and runs its code once on no cells while it waits, to cache the instructions.
cudaError_t launch_attend_selected(const LayerView& L, const void* q, const int32_t* sel,
                                   const int32_t* n_sel, float* out, cudaStream_t s, int n_queries = 1,
                                   float* lse = nullptr, bool warm = false);
// context-parallel step (qsa_cp.cu)
cudaError_t launch_cp_select(const float* cand_scores, const int32_t* cand_blocks, int n_shards, int k_blocks,
                             int32_t* sel, int32_t* n_sel, cudaStream_t s);
cudaError_t launch_cp_filter(const LayerView& L, const int32_t* sel_global, const int32_t* n_sel_global,
                             int block_base, int32_t* sel_local, int32_t* n_local, cudaStream_t s);
cudaError_t launch_cp_merge(const float* o_parts, const float* lse_parts, int n_shards, int n_q_heads, int head_dim,
                            float* out, cudaStream_t s);
cudaError_t launch_attend_split(const LayerView& L, const void* q, const int32_t* cells,
                                const int32_t* n_cells, float* out, cudaStream_t s);
cudaError_t plan_attention(const qsa_config& c, int* cluster, int* cells_per_cta);

// set_state modes
enum { kSetReset = 0, kSetRestore = 1, kSetInvalidate = 2, kSetClearStatus = 3, kSetRollback = 4 };

}  // namespace qsa
