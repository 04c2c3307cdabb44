// C ABI of the QSA decode hot path: host-side validation, the host context and the
// dispatch of each call to its kernels. The device-side sequence state lives in the
// layer workspace (see qsa_internal.h); nothing here allocates device memory.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "../../include/qsa.h"
#include "qsa_internal.h"

using namespace qsa;

static_assert(QSA_MAX_QUERIES == kMaxQueries, "header and kernels agree on the multi-query limit");

namespace {

struct Layer {
  bool bound = false;
  qsa_layer_buffers buf{};
  CUtensorMap pooled_tile_map{}, pooled_box_map{};
  // Upper bound on blocks the next pooled update may have to compute; it only sizes
  // the update's grid (the kernel itself reads the exact range from device state).
  long long pending_blocks = 0;
};

bool is_pow2_upto(int v, int hi) { return v >= 1 && v <= hi && (v & (v - 1)) == 0; }

const char* config_problem(const qsa_config& c) {
  if (c.n_layers < 1) return "n_layers must be >= 1";
  if (c.max_ctx < kBlock || c.max_ctx % kBlock) return "max_ctx must be a positive multiple of 4";
  if (c.max_ctx > kBlock * kTopkCluster * kTopkMaxPerCta) return "max_ctx above 1,048,576";
  if (c.d_idx != 64 && c.d_idx != 128) return "d_idx must be 64 or 128";
  if (!is_pow2_upto(c.n_idx_heads, 16)) return "n_idx_heads must be 1, 2, 4, 8 or 16";
  if (c.top_k_tokens < kBlock || c.top_k_tokens % kBlock) return "top_k_tokens must be a positive multiple of 4";
  // the attention cluster stages at most 16 x 256 cells: K blocks plus the 3-token tail
  if (c.top_k_tokens > 4092 || c.top_k_tokens / kBlock > kTopkMaxK) return "top_k_tokens above 4092";
  if (c.head_dim != 64 && c.head_dim != 128) return "head_dim must be 64 or 128";
  if (c.n_kv_heads < 1 || c.n_q_heads < 1 || c.n_q_heads % c.n_kv_heads) return "n_q_heads must be a multiple of n_kv_heads";
  if (!is_pow2_upto(c.n_q_heads / c.n_kv_heads, 8)) return "n_q_heads / n_kv_heads must be 1, 2, 4 or 8";
  if (!(c.rope_base > 1.0f)) return "rope_base must be > 1";
  if (!(c.rms_eps >= 0.0f)) return "rms_eps must be >= 0";
  if (c.rope_dims < 0 || c.rope_dims > c.d_idx || c.rope_dims % 2) return "rope_dims must be even and <= d_idx";
  if (c.rope_interleaved != 0 && c.rope_interleaved != 1) return "rope_interleaved must be 0 or 1";
  if (c.rope_pos_stride < 0 || c.rope_pos_stride > 16) return "rope_pos_stride must be 0..16";
  if (c.rope_pos_offset < 0 || c.rope_pos_offset > (1 << 20)) return "rope_pos_offset must be 0..1048576";
  if (c.kv_format != QSA_KV_F16 && c.kv_format != QSA_KV_FP8) return "kv_format must be QSA_KV_F16 or QSA_KV_FP8";
  if (c.scan_kind != QSA_SCAN_TENSOR && c.scan_kind != QSA_SCAN_CUDA_CORES)
    return "scan_kind must be QSA_SCAN_TENSOR or QSA_SCAN_CUDA_CORES";
  if (c.pooled_format != QSA_POOLED_F16 && c.pooled_format != QSA_POOLED_FP8)
    return "pooled_format must be QSA_POOLED_F16 or QSA_POOLED_FP8";
  if (c.pooled_format == QSA_POOLED_FP8 && (c.d_idx != 128 || c.scan_kind != QSA_SCAN_TENSOR))
    return "QSA_POOLED_FP8 needs d_idx 128 and the tensor-core scan";
  if (c.early_inputs != QSA_INPUTS_ORDERED && c.early_inputs != QSA_INPUTS_EARLY)
    return "early_inputs must be QSA_INPUTS_ORDERED or QSA_INPUTS_EARLY";
  return nullptr;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

struct qsa_ctx {
  qsa_config cfg{};
  int device = 0;
  int n_sms = 0;
  AttnSplit split{};
  int attn_cluster = 0, attn_cells_per_cta = 0;
  WorkspaceLayout ws{};
  std::vector<Layer> layers;
  std::string last_error;

  qsa_status fail(qsa_status st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    last_error = buf;
    return st;
  }
  qsa_status cuda(cudaError_t e, const char* what) {
    if (e == cudaSuccess) return QSA_OK;
    return fail(QSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  }
  qsa_status layer_ok(int32_t layer) {
    if (layer < 0 || layer >= cfg.n_layers) return fail(QSA_ERR_INVALID_ARG, "layer %d out of range", layer);
    if (!layers[layer].bound) return fail(QSA_ERR_STATE, "layer %d has no buffers bound", layer);
    return QSA_OK;
  }
  LayerView view(int32_t layer) const {
    const Layer& l = layers[layer];
    char* wsp = static_cast<char*>(l.buf.workspace);
    LayerView v;
    v.cfg = cfg;
    v.k_cache = l.buf.k_cache;
    v.v_cache = l.buf.v_cache;
    v.idx_cache = l.buf.idx_cache;
    v.pooled_cache = l.buf.pooled_cache;
    v.rms_gain = l.buf.rms_gain;
    v.kv_scales = static_cast<float*>(l.buf.kv_scales);
    v.pooled_scales = static_cast<float*>(l.buf.pooled_scales);
    v.state = reinterpret_cast<DevState*>(wsp + ws.state);
    v.scores = reinterpret_cast<float*>(wsp + ws.scores);
    v.hist = reinterpret_cast<uint32_t*>(wsp + ws.hist);
    v.cp_count = reinterpret_cast<int32_t*>(wsp + ws.cp);
    v.cp_sel = v.cp_count + 16;
    v.part_o = reinterpret_cast<float*>(wsp + ws.part_o);
    v.part_ml = reinterpret_cast<float*>(wsp + ws.part_ml);
    v.split = split;
    v.n_sms = n_sms;
    v.pooled_tile_map = l.pooled_tile_map;
    v.pooled_box_map = l.pooled_box_map;
    v.attn_cluster = attn_cluster;
    v.attn_cells_per_cta = attn_cells_per_cta;
    return v;
  }
};

#define QSA_CHECK_PTR(p, a, name)                                                         \
  do {                                                                                    \
    if (!(p) || !aligned((p), (a)))                                                       \
      return ctx->fail(QSA_ERR_INVALID_ARG, "%s must be a non-null %d-byte aligned pointer", \
                       name, (int)(a));                                                   \
  } while (0)

extern "C" {

size_t qsa_buffer_bytes(const qsa_config* cfg, int32_t which) {
  if (!cfg || config_problem(*cfg)) return 0;
  const qsa_config& c = *cfg;
  switch (which) {
    case QSA_BUF_KV: return size_t(c.max_ctx) * c.n_kv_heads * c.head_dim * (c.kv_format == QSA_KV_FP8 ? 1 : 2);
    case QSA_BUF_KV_SCALES: return c.kv_format == QSA_KV_FP8 ? size_t(c.max_ctx) * c.n_kv_heads * 2 * 4 : 0;
    case QSA_BUF_IDX: return size_t(c.max_ctx) * c.d_idx * 2;
    case QSA_BUF_POOLED: return size_t(c.max_ctx / kBlock) * c.d_idx * (c.pooled_format == QSA_POOLED_FP8 ? 1 : 2);
    case QSA_BUF_POOLED_SCALES: return c.pooled_format == QSA_POOLED_FP8 ? size_t(c.max_ctx / kBlock) * 4 : 0;
    case QSA_BUF_WORKSPACE: {
      int dev = 0, sms = 0;
      if (cudaGetDevice(&dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
        sms = 148;
      // the largest split count any device could choose (one SM per CTA)
      const AttnSplit worst = attn_split(c, sms > 148 ? sms : 148);
      const AttnSplit here = attn_split(c, sms);
      const int n_splits = worst.n_splits > here.n_splits ? worst.n_splits : here.n_splits;
      return workspace_layout(c, n_splits).total;
    }
    case QSA_BUF_MAX_CELLS: return size_t(max_cells_of(c));
    case QSA_BUF_SCORE_STRIDE: return size_t(score_stride_of(c));
    default: return 0;
  }
}

qsa_status qsa_create(const qsa_config* cfg, qsa_ctx** out) {
  if (!cfg || !out) return QSA_ERR_INVALID_ARG;
  *out = nullptr;
  if (config_problem(*cfg)) return QSA_ERR_UNSUPPORTED;
  qsa_ctx* ctx = new (std::nothrow) qsa_ctx();
  if (!ctx) return QSA_ERR_INVALID_ARG;
  ctx->cfg = *cfg;
  if (ctx->cfg.rope_dims == 0) ctx->cfg.rope_dims = ctx->cfg.d_idx;  // zero fields take the defaults
  if (ctx->cfg.rope_pos_stride == 0) ctx->cfg.rope_pos_stride = kBlock;
  if (cudaGetDevice(&ctx->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&ctx->n_sms, cudaDevAttrMultiProcessorCount, ctx->device) != cudaSuccess) {
    delete ctx;
    return QSA_ERR_CUDA;
  }
  if (init_kernel_attributes() != cudaSuccess || init_scan_attributes() != cudaSuccess ||
      init_scan_cc_attributes() != cudaSuccess) {
    delete ctx;
    return QSA_ERR_CUDA;
  }
  if (plan_attention(*cfg, &ctx->attn_cluster, &ctx->attn_cells_per_cta) != cudaSuccess) {
    delete ctx;
    return QSA_ERR_UNSUPPORTED;
  }
  ctx->split = attn_split(*cfg, ctx->n_sms);
  const AttnSplit worst = attn_split(*cfg, ctx->n_sms > 148 ? ctx->n_sms : 148);
  ctx->ws = workspace_layout(*cfg, worst.n_splits > ctx->split.n_splits ? worst.n_splits : ctx->split.n_splits);
  ctx->layers.resize(cfg->n_layers);
  *out = ctx;
  return QSA_OK;
}

void qsa_destroy(qsa_ctx* ctx) { delete ctx; }

const char* qsa_last_error(const qsa_ctx* ctx) { return ctx ? ctx->last_error.c_str() : "null context"; }

qsa_status qsa_bind_layer(qsa_ctx* ctx, int32_t layer, const qsa_layer_buffers* buf, qsa_stream_t stream) {
  if (!ctx) return QSA_ERR_INVALID_ARG;
  if (!buf) return ctx->fail(QSA_ERR_INVALID_ARG, "buffers must not be null");
  if (layer < 0 || layer >= ctx->cfg.n_layers) return ctx->fail(QSA_ERR_INVALID_ARG, "layer %d out of range", layer);
  QSA_CHECK_PTR(buf->k_cache, 16, "k_cache");
  QSA_CHECK_PTR(buf->v_cache, 16, "v_cache");
  QSA_CHECK_PTR(buf->idx_cache, 16, "idx_cache");
  QSA_CHECK_PTR(buf->pooled_cache, 16, "pooled_cache");
  QSA_CHECK_PTR(buf->workspace, 256, "workspace");
  if (buf->rms_gain && !aligned(buf->rms_gain, 16))
    return ctx->fail(QSA_ERR_INVALID_ARG, "rms_gain must be 16-byte aligned");
  if (ctx->cfg.kv_format == QSA_KV_FP8) QSA_CHECK_PTR(buf->kv_scales, 16, "kv_scales");
  if (ctx->cfg.pooled_format == QSA_POOLED_FP8) QSA_CHECK_PTR(buf->pooled_scales, 16, "pooled_scales");
  Layer& l = ctx->layers[layer];
  CUtensorMap tile_map, box_map;
  if (qsa_status st = ctx->cuda(encode_pooled_map(ctx->cfg, buf->pooled_cache, 128, &tile_map), "bind_layer: pooled TMA map"))
    return st;
  if (qsa_status st = ctx->cuda(encode_pooled_map(ctx->cfg, buf->pooled_cache, 16, &box_map), "bind_layer: pooled TMA map"))
    return st;
  l.buf = *buf;
  l.pooled_tile_map = tile_map;
  l.pooled_box_map = box_map;
  l.bound = true;
  l.pending_blocks = 0;
  const LayerView v = ctx->view(layer);
  qsa_status st = ctx->cuda(cudaMemsetAsync(v.hist, 0, size_t(kMaxQueries) * (1 << kHistBits) * sizeof(uint32_t),
                                            (cudaStream_t)stream),
                            "bind_layer: clear histogram");
  if (st == QSA_OK) st = ctx->cuda(launch_set_state(v, 0, 0, kSetReset, (cudaStream_t)stream), "bind_layer");
  if (st != QSA_OK) l.bound = false;
  return st;
}

qsa_status qsa_restore_layer(qsa_ctx* ctx, int32_t layer, int32_t n_ctx, int32_t n_pooled, qsa_stream_t stream) {
  if (!ctx) return QSA_ERR_INVALID_ARG;
  if (qsa_status st = ctx->layer_ok(layer)) return st;
  if (n_ctx < 0 || n_ctx > ctx->cfg.max_ctx)
    return ctx->fail(QSA_ERR_CAPACITY, "n_ctx %d outside [0, max_ctx=%d]", n_ctx, ctx->cfg.max_ctx);
  if (n_pooled < 0 || n_pooled > n_ctx / kBlock)
    return ctx->fail(QSA_ERR_INVALID_ARG, "n_pooled %d outside [0, n_ctx/4]", n_pooled);
  ctx->layers[layer].pending_blocks = n_ctx / kBlock - n_pooled;
  return ctx->cuda(launch_set_state(ctx->view(layer), n_ctx, n_pooled, kSetRestore, (cudaStream_t)stream),
                   "restore_layer");
}

qsa_status qsa_read_layer_state(qsa_ctx* ctx, int32_t layer, int32_t* n_ctx, int32_t* n_pooled,
                                int32_t* device_status, int32_t clear, qsa_stream_t stream) {
  if (!ctx) return QSA_ERR_INVALID_ARG;
  if (qsa_status st = ctx->layer_ok(layer)) return st;
  LayerView v = ctx->view(layer);
  if (qsa_status st = ctx->cuda(cudaStreamSynchronize((cudaStream_t)stream), "read_layer_state: sync")) return st;
  DevState h;
  if (qsa_status st = ctx->cuda(cudaMemcpy(&h, v.state, sizeof h, cudaMemcpyDeviceToHost), "read_layer_state: copy"))
    return st;
  if (n_ctx) *n_ctx = h.n_ctx;
  if (n_pooled) *n_pooled = h.n_pooled;
  if (device_status) *device_status = h.status;
  if (clear) {
    if (qsa_status st = ctx->cuda(launch_set_state(v, 0, 0, kSetClearStatus, (cudaStream_t)stream), "clear status"))
      return st;
    return ctx->cuda(cudaStreamSynchronize((cudaStream_t)stream), "read_layer_state: sync");
  }
  return QSA_OK;
}

qsa_status qsa_append_tokens(qsa_ctx* ctx, int32_t layer, int32_t n, const void* k, const void* v,
                             const void* idx_key, qsa_stream_t stream) {
  if (!ctx) return QSA_ERR_INVALID_ARG;
  if (qsa_status st = ctx->layer_ok(layer)) return st;
  if (n < 1 || n > ctx->cfg.max_ctx) return ctx->fail(QSA_ERR_CAPACITY, "cannot append %d tokens", n);
  QSA_CHECK_PTR(k, 16, "k");
  QSA_CHECK_PTR(v, 16, "v");
  QSA_CHECK_PTR(idx_key, 16, "idx_key");
  Layer& l = ctx->layers[layer];
  l.pending_blocks += n / kBlock + 1;
  if (l.pending_blocks > ctx->cfg.max_ctx / kBlock) l.pending_blocks = ctx->cfg.max_ctx / kBlock;
  return ctx->cuda(launch_append(ctx->view(layer), n, k, v, idx_key, ctx->n_sms * 4, (cudaStream_t)stream),
                   "append_tokens");
}

qsa_status qsa_append_token(qsa_ctx* ctx, int32_t layer, const void* k, const void* v, const void* idx_key,
                            qsa_stream_t stream) {
  return qsa_append_tokens(ctx, layer, 1, k, v, idx_key, stream);
}

qsa_status qsa_decode_append(qsa_ctx* ctx, int32_t layer, const void* k, const void* v, const void* idx_key,
                             qsa_stream_t stream) {
  if (!ctx) return QSA_ERR_INVALID_ARG;
  if (qsa_status st = ctx->layer_ok(layer)) return st;
  QSA_CHECK_PTR(k, 16, "k");
  QSA_CHECK_PTR(v, 16, "v");
  QSA_CHECK_PTR(idx_key, 16, "idx_key");
  qsa_status st = ctx->cuda(launch_decode_append(ctx->view(layer), k, v, idx_key, (cudaStream_t)stream),
                            "decode_append");
  if (st == QSA_OK) ctx->layers[layer].pending_blocks = 0;  // the call pools every completed block
  return st;
}

qsa_status qsa_update_pooled_cache(qsa_ctx* ctx, int32_t layer, qsa_stream_t stream) {
  if (!ctx) return QSA_ERR_INVALID_ARG;
  if (qsa_status st = ctx->layer_ok(layer)) return st;
  Layer& l = ctx->layers[layer];
  // 8 warps per CTA, 4 blocks per warp per round; at most ~4 resident CTAs per SM
  long long grid = (l.pending_blocks + 31) / 32;
  if (grid < 1) grid = 1;
  if (grid > ctx->n_sms * 4) grid = ctx->n_sms * 4;
  l.pending_blocks = 0;
  return ctx->cuda(launch_pool_update(ctx->view(layer), (int)grid, (cudaStream_t)stream), "update_pooled_cache");
}

qsa_status qsa_invalidate_pooled_cache(qsa_ctx* ctx, int32_t layer, int32_t from_block, qsa_stream_t stream) {
  if (!ctx) return QSA_ERR_INVALID_ARG;
  if (qsa_status st = ctx->layer_ok(layer)) return st;
  if (from_block < 0) return ctx->fail(QSA_ERR_INVALID_ARG, "from_block must be >= 0");
  Layer& l = ctx->layers[layer];
  l.pending_blocks = ctx->cfg.max_ctx / kBlock - (from_block < ctx->cfg.max_ctx / kBlock ? from_block : 0);
  return ctx->cuda(launch_set_state(ctx->view(layer), 0, from_block, kSetInvalidate, (cudaStream_t)stream),
                   "invalidate_pooled_cache");
}

qsa_status qsa_index_topk(qsa_ctx* ctx, int32_t layer, const void* q_idx, const float* w, int32_t* sel_blocks,
                          int32_t* n_sel, float* scores, qsa_stream_t stream) {
  if (!ctx) return QSA_ERR_INVALID_ARG;
  if (qsa_status st = ctx->layer_ok(layer)) return st;
  QSA_CHECK_PTR(q_idx, 16, "q_idx");
  QSA_CHECK_PTR(w, 16, "w");
  QSA_CHECK_PTR(sel_blocks, 16, "sel_blocks");
  QSA_CHECK_PTR(n_sel, 4, "n_sel");
  if (scores && !aligned(scores, 16)) return ctx->fail(QSA_ERR_INVALID_ARG, "scores must be 16-byte aligned");
  LayerView v = ctx->view(layer);
  float* s = scores ? scores : v.scores;
  // the scan fills the score-key histogram the selection starts from (and clears)
  if (qsa_status st = ctx->cuda(launch_index_scan(v, q_idx, w, s, (cudaStream_t)stream, 1, 0, v.hist), "index scan"))
    return st;
  return ctx->cuda(launch_topk(v, s, sel_blocks, n_sel, (cudaStream_t)stream, 1, 0, v.hist), "block top-k");
}

qsa_status qsa_index_scores(qsa_ctx* ctx, int32_t layer, const void* q_idx, const float* w, float* scores,
                            qsa_stream_t stream) {
  if (!ctx) return QSA_ERR_INVALID_ARG;
  if (qsa_status st = ctx->layer_ok(layer)) return st;
  QSA_CHECK_PTR(q_idx, 16, "q_idx");
  QSA_CHECK_PTR(w, 16, "w");
  QSA_CHECK_PTR(scores, 16, "scores");
  return ctx->cuda(launch_index_scan(ctx->view(layer), q_idx, w, scores, (cudaStream_t)stream), "index scan");
}

qsa_status qsa_select_topk(qsa_ctx* ctx, int32_t layer, const float* scores, int32_t* sel_blocks, int32_t* n_sel,
                           qsa_stream_t stream) {
  if (!ctx) return QSA_ERR_INVALID_ARG;
  if (qsa_status st = ctx->layer_ok(layer)) return st;
  QSA_CHECK_PTR(scores, 16, "scores");
  QSA_CHECK_PTR(sel_blocks, 16, "sel_blocks");
  QSA_CHECK_PTR(n_sel, 4, "n_sel");
  return ctx->cuda(launch_topk(ctx->view(layer), scores, sel_blocks, n_sel, (cudaStream_t)stream), "block top-k");
}

qsa_status qsa_gather_kv(qsa_ctx* ctx, int32_t layer, const int32_t* sel_blocks, const int32_t* n_sel,
                         int32_t* cells, int32_t* n_cells, void* k_compact, void* v_compact, qsa_stream_t stream) {
  if (!ctx) return QSA_ERR_INVALID_ARG;
  if (qsa_status st = ctx->layer_ok(layer)) return st;
  QSA_CHECK_PTR(sel_blocks, 16, "sel_blocks");
  QSA_CHECK_PTR(n_sel, 4, "n_sel");
  QSA_CHECK_PTR(cells, 16, "cells");
  QSA_CHECK_PTR(n_cells, 4, "n_cells");
  if ((k_compact && !aligned(k_compact, 16)) || (v_compact && !aligned(v_compact, 16)))
    return ctx->fail(QSA_ERR_INVALID_ARG, "compact K/V must be 16-byte aligned");
  if ((k_compact || v_compact) && ctx->cfg.kv_format == QSA_KV_FP8)
    return ctx->fail(QSA_ERR_UNSUPPORTED, "compact K/V copies need an f16 K/V cache");
  return ctx->cuda(launch_gather(ctx->view(layer), sel_blocks, n_sel, cells, n_cells, k_compact, v_compact,
                                 (cudaStream_t)stream),
                   "gather_kv");
}

qsa_status qsa_sparse_attend(qsa_ctx* ctx, int32_t layer, const void* q, const int32_t* cells,
                             const int32_t* n_cells, float* out, qsa_stream_t stream) {
  if (!ctx) return QSA_ERR_INVALID_ARG;
  if (qsa_status st = ctx->layer_ok(layer)) return st;
  QSA_CHECK_PTR(q, 16, "q");
  QSA_CHECK_PTR(cells, 16, "cells");
  QSA_CHECK_PTR(n_cells, 4, "n_cells");
  QSA_CHECK_PTR(out, 16, "out");
  return ctx->cuda(launch_attend(ctx->view(layer), q, cells, n_cells, out, (cudaStream_t)stream), "sparse_attend");
}

qsa_status qsa_index_topk_multi(qsa_ctx* ctx, int32_t layer, int32_t n_queries, const void* q_idx, const float* w,
                                int32_t* sel_blocks, int32_t* n_sel, float* scores, qsa_stream_t stream) {
  if (!ctx) return QSA_ERR_INVALID_ARG;
  if (qsa_status st = ctx->layer_ok(layer)) return st;
  if (n_queries < 1 || n_queries > kMaxQueries)
    return ctx->fail(QSA_ERR_INVALID_ARG, "n_queries %d outside [1, %d]", n_queries, kMaxQueries);
  if (n_queries > 1 && ctx->cfg.pooled_format == QSA_POOLED_FP8)
    return ctx->fail(QSA_ERR_UNSUPPORTED, "8-bit pooled keys are scanned one query at a time");
  QSA_CHECK_PTR(q_idx, 16, "q_idx");
  QSA_CHECK_PTR(w, 4, "w");
  QSA_CHECK_PTR(sel_blocks, 16, "sel_blocks");
  QSA_CHECK_PTR(n_sel, 4, "n_sel");
  if (scores && !aligned(scores, 16)) return ctx->fail(QSA_ERR_INVALID_ARG, "scores must be 16-byte aligned");
  LayerView v = ctx->view(layer);
  const int stride = score_stride_of(ctx->cfg);
  float* s = scores ? scores : v.scores;
  if (qsa_status st = ctx->cuda(launch_index_scan(v, q_idx, w, s, (cudaStream_t)stream, n_queries, stride, v.hist),
                                "index scan (multi-query)"))
    return st;
  return ctx->cuda(launch_topk(v, s, sel_blocks, n_sel, (cudaStream_t)stream, n_queries, stride, v.hist),
                   "block top-k (multi-query)");
}

qsa_status qsa_sparse_attend_selected_multi(qsa_ctx* ctx, int32_t layer, int32_t n_queries, const void* q,
                                            const int32_t* sel_blocks, const int32_t* n_sel, float* out,
                                            qsa_stream_t stream) {
  if (!ctx) return QSA_ERR_INVALID_ARG;
  if (qsa_status st = ctx->layer_ok(layer)) return st;
  if (n_queries < 1 || n_queries > kMaxQueries)
    return ctx->fail(QSA_ERR_INVALID_ARG, "n_queries %d outside [1, %d]", n_queries, kMaxQueries);
  QSA_CHECK_PTR(q, 16, "q");
  QSA_CHECK_PTR(sel_blocks, 16, "sel_blocks");
  QSA_CHECK_PTR(n_sel, 4, "n_sel");
  QSA_CHECK_PTR(out, 16, "out");
  return ctx->cuda(launch_attend_selected(ctx->view(layer), q, sel_blocks, n_sel, out, (cudaStream_t)stream,
                                          n_queries),
                   "sparse_attend_selected (multi-query)");
}

size_t qsa_layer_bytes(const qsa_config* cfg, int32_t which) { return qsa_buffer_bytes(cfg, which); }

int32_t qsa_n_ctx(const qsa_ctx* ctx, int32_t layer) {
  if (!ctx || layer < 0 || layer >= ctx->cfg.n_layers || !ctx->layers[layer].bound) return -1;
  if (cudaDeviceSynchronize() != cudaSuccess) return -1;
  DevState h;
  if (cudaMemcpy(&h, ctx->view(layer).state, sizeof h, cudaMemcpyDeviceToHost) != cudaSuccess) return -1;
  return h.n_ctx;
}

qsa_status qsa_get_device_status(qsa_ctx* ctx, int32_t* status_out) {
  if (!ctx || !status_out) return QSA_ERR_INVALID_ARG;
  *status_out = QSA_OK;
  if (qsa_status st = ctx->cuda(cudaDeviceSynchronize(), "get_device_status: sync")) return st;
  for (int32_t layer = 0; layer < ctx->cfg.n_layers; ++layer) {
    if (!ctx->layers[layer].bound) continue;
    DevState h;
    if (qsa_status st = ctx->cuda(cudaMemcpy(&h, ctx->view(layer).state, sizeof h, cudaMemcpyDeviceToHost),
                                  "get_device_status: copy"))
      return st;
    if (h.status != 0) {
      *status_out = h.status;
      break;
    }
  }
  return QSA_OK;
}

qsa_status qsa_decode_step(qsa_ctx* ctx, int32_t layer, const void* k, const void* v, const void* idx_key,
                           const void* q_idx, const float* w, const void* q, int32_t* sel_blocks, int32_t* n_sel,
                           float* out, qsa_stream_t stream) {
  if (!ctx) return QSA_ERR_INVALID_ARG;
  if (qsa_status st = ctx->layer_ok(layer)) return st;
  QSA_CHECK_PTR(k, 16, "k");
  QSA_CHECK_PTR(v, 16, "v");
  QSA_CHECK_PTR(idx_key, 16, "idx_key");
  QSA_CHECK_PTR(q_idx, 16, "q_idx");
  QSA_CHECK_PTR(w, 4, "w");
  QSA_CHECK_PTR(q, 16, "q");
  QSA_CHECK_PTR(sel_blocks, 16, "sel_blocks");
  QSA_CHECK_PTR(n_sel, 4, "n_sel");
  QSA_CHECK_PTR(out, 16, "out");
  const LayerView lv = ctx->view(layer);
  const cudaStream_t s = (cudaStream_t)stream;
  Layer& l = ctx->layers[layer];
  const bool fused = l.pending_blocks == 0 && ctx->cfg.scan_kind == QSA_SCAN_TENSOR;
  if (fused) {
    // the pooled cache is current up to the previous token: the scan kernel itself
    // appends the token and pools the block it completes (three launches per step); the
    // selection then advances the state past the token
    if (qsa_status st = ctx->cuda(launch_decode_scan(lv, k, v, idx_key, q_idx, w, lv.scores, lv.hist, s),
                                  "decode_step: append + index scan"))
      return st;
  } else {
    // blocks are waiting to be pooled (after a bulk append or an invalidation), or the
    // layer scans on the CUDA cores: the separate append pools every waiting block first
    if (qsa_status st = ctx->cuda(launch_decode_append(lv, k, v, idx_key, s), "decode_step: append")) return st;
    l.pending_blocks = 0;
    if (qsa_status st = ctx->cuda(launch_index_scan(lv, q_idx, w, lv.scores, s, 1, 0, lv.hist),
                                  "decode_step: index scan"))
      return st;
  }
  if (qsa_status st = ctx->cuda(launch_topk(lv, lv.scores, sel_blocks, n_sel, s, 1, 0, lv.hist, nullptr, 0, fused),
                                "decode_step: block top-k"))
    return st;
  return ctx->cuda(launch_attend_selected(lv, q, sel_blocks, n_sel, out, s, 1, nullptr, true),
                   "decode_step: sparse attend");
}

qsa_status qsa_rollback(qsa_ctx* ctx, int32_t layer, int32_t n_keep, qsa_stream_t stream) {
  if (!ctx) return QSA_ERR_INVALID_ARG;
  if (qsa_status st = ctx->layer_ok(layer)) return st;
  if (n_keep < 0) return ctx->fail(QSA_ERR_INVALID_ARG, "n_keep must be >= 0");
  // Dropping tokens never adds blocks to pool: the kept summaries [0, n_keep/4) stay valid
  // and the pooled count is cut to them, so the count of blocks waiting to be pooled can
  // only fall (pending_blocks stays an upper bound).
  return ctx->cuda(launch_set_state(ctx->view(layer), n_keep, 0, kSetRollback, (cudaStream_t)stream), "rollback");
}

qsa_status qsa_cp_index_candidates(qsa_ctx* ctx, int32_t layer, const void* q_idx, const float* w, int32_t n_global,
                                   int32_t block_base, float* cand_scores, int32_t* cand_blocks, int32_t* n_cand,
                                   qsa_stream_t stream) {
  if (!ctx) return QSA_ERR_INVALID_ARG;
  if (qsa_status st = ctx->layer_ok(layer)) return st;
  QSA_CHECK_PTR(q_idx, 16, "q_idx");
  QSA_CHECK_PTR(w, 4, "w");
  QSA_CHECK_PTR(cand_scores, 16, "cand_scores");
  QSA_CHECK_PTR(cand_blocks, 16, "cand_blocks");
  QSA_CHECK_PTR(n_cand, 4, "n_cand");
  if (n_global < 1) return ctx->fail(QSA_ERR_INVALID_ARG, "n_global must be >= 1");
  if (block_base < 0) return ctx->fail(QSA_ERR_INVALID_ARG, "block_base must be >= 0");
  const LayerView v = ctx->view(layer);
  const cudaStream_t s = (cudaStream_t)stream;
  if (qsa_status st = ctx->cuda(launch_index_scan(v, q_idx, w, v.scores, s, 1, 0, v.hist, n_global),
                                "cp_index_candidates: index scan"))
    return st;
  return ctx->cuda(launch_topk(v, v.scores, cand_blocks, n_cand, s, 1, 0, v.hist, cand_scores, block_base),
                   "cp_index_candidates: local top-k");
}

qsa_status qsa_cp_attend_partial(qsa_ctx* ctx, int32_t layer, const void* q, const int32_t* sel_blocks,
                                 const int32_t* n_sel, int32_t block_base, float* out, float* lse,
                                 qsa_stream_t stream) {
  if (!ctx) return QSA_ERR_INVALID_ARG;
  if (qsa_status st = ctx->layer_ok(layer)) return st;
  QSA_CHECK_PTR(q, 16, "q");
  QSA_CHECK_PTR(sel_blocks, 4, "sel_blocks");
  QSA_CHECK_PTR(n_sel, 4, "n_sel");
  QSA_CHECK_PTR(out, 16, "out");
  QSA_CHECK_PTR(lse, 4, "lse");
  if (block_base < 0) return ctx->fail(QSA_ERR_INVALID_ARG, "block_base must be >= 0");
  const LayerView v = ctx->view(layer);
  const cudaStream_t s = (cudaStream_t)stream;
  if (qsa_status st = ctx->cuda(launch_cp_filter(v, sel_blocks, n_sel, block_base, v.cp_sel, v.cp_count, s),
                                "cp_attend_partial: this shard's blocks"))
    return st;
  return ctx->cuda(launch_attend_selected(v, q, v.cp_sel, v.cp_count, out, s, 1, lse), "cp_attend_partial: attend");
}

qsa_status qsa_cp_select(const float* cand_scores, const int32_t* cand_blocks, int32_t n_shards, int32_t k_blocks,
                         int32_t* sel_blocks, int32_t* n_sel, qsa_stream_t stream) {
  if (!cand_scores || !cand_blocks || !sel_blocks || !n_sel || !aligned(cand_scores, 4) || !aligned(cand_blocks, 4) ||
      !aligned(sel_blocks, 4) || !aligned(n_sel, 4))
    return QSA_ERR_INVALID_ARG;
  if (n_shards < 1 || k_blocks < 1 || k_blocks > kTopkMaxK) return QSA_ERR_INVALID_ARG;
  if (n_shards * k_blocks > 8192) return QSA_ERR_UNSUPPORTED;
  return launch_cp_select(cand_scores, cand_blocks, n_shards, k_blocks, sel_blocks, n_sel, (cudaStream_t)stream) ==
                 cudaSuccess
             ? QSA_OK
             : QSA_ERR_CUDA;
}

qsa_status qsa_cp_merge(const float* o_parts, const float* lse_parts, int32_t n_shards, int32_t n_q_heads,
                        int32_t head_dim, float* out, qsa_stream_t stream) {
  if (!o_parts || !lse_parts || !out || !aligned(o_parts, 4) || !aligned(lse_parts, 4) || !aligned(out, 4))
    return QSA_ERR_INVALID_ARG;
  if (n_shards < 1 || n_q_heads < 1 || head_dim < 1) return QSA_ERR_INVALID_ARG;
  return launch_cp_merge(o_parts, lse_parts, n_shards, n_q_heads, head_dim, out, (cudaStream_t)stream) == cudaSuccess
             ? QSA_OK
             : QSA_ERR_CUDA;
}

qsa_status qsa_sparse_attend_selected(qsa_ctx* ctx, int32_t layer, const void* q, const int32_t* sel_blocks,
                                      const int32_t* n_sel, float* out, qsa_stream_t stream) {
  if (!ctx) return QSA_ERR_INVALID_ARG;
  if (qsa_status st = ctx->layer_ok(layer)) return st;
  QSA_CHECK_PTR(q, 16, "q");
  QSA_CHECK_PTR(sel_blocks, 16, "sel_blocks");
  QSA_CHECK_PTR(n_sel, 4, "n_sel");
  QSA_CHECK_PTR(out, 16, "out");
  return ctx->cuda(launch_attend_selected(ctx->view(layer), q, sel_blocks, n_sel, out, (cudaStream_t)stream),
                   "sparse_attend_selected");
}

}  // extern "C"
