// Sequence state, token append and the incremental pooled-key cache.
//
// Incremental pooled-key cache: web page "Part 10" (第10回 EVO-X2 ... 長コンテキストのTGを
// 高速化した話), section "incremental pooled-key cache（COMMON-004）": completed-block
// summaries are kept per layer and only blocks that completed (or were invalidated)
// since the last update are computed. Summary of block b (section "QSA indexer"):
// mean of its 4 raw indexer keys -> RMS norm -> RoPE at the block position, stored
// as f16. RoPE is by default the NeoX half-split rotation of pair (i, i+d/2) by angle
// pos * base^(-2i/d), with the block at position 4b; the layer config can narrow the
// rotary dims, pair adjacent elements instead, or rescale and shift block positions.
// Angles are reduced in double precision so that positions near 2.6e5 keep full
// accuracy; the rotation itself runs in f32.
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "qsa_checked.cuh"
#include "qsa_device.cuh"
#include "qsa_pool.cuh"

namespace qsa {

__global__ void set_state_kernel(DevState* st, int n_ctx, int n_pooled, int mode) {
  pdl_launch_dependents();
  pdl_wait();
  if (threadIdx.x != 0) return;
  if (mode == kSetReset) {
    st->n_ctx = 0;
    st->n_pooled = 0;
    st->status = 0;
    st->ticket_append = 0;
    st->ticket_pool = 0;
  } else if (mode == kSetRestore) {
    st->n_ctx = n_ctx;
    st->n_pooled = n_pooled;
    st->status = 0;
    st->ticket_append = 0;
    st->ticket_pool = 0;
  } else if (mode == kSetInvalidate) {
    if (st->n_pooled > n_pooled) st->n_pooled = n_pooled;
  } else if (mode == kSetRollback) {  // drop tokens >= n_ctx and the blocks they completed
    if (st->n_ctx > n_ctx) st->n_ctx = n_ctx;
    if (st->n_pooled > st->n_ctx / kBlock) st->n_pooled = st->n_ctx / kBlock;
  } else {
    st->status = 0;
  }
}

cudaError_t launch_set_state(const LayerView& L, int n_ctx, int n_pooled, int mode, cudaStream_t s) {
  return launch_pdl(set_state_kernel, dim3(1), dim3(32), 0, s, 1, L.state, n_ctx, n_pooled, mode);
}

// Appends n tokens at position n_ctx: three contiguous copies (token-major caches), in
// 16-byte units (FP8: the K/V rows quantised a warp per row). All CTAs read n_ctx before
// any of them can change it: the last CTA to finish (atomic ticket) publishes n_ctx + n.
template <bool FP8>
__global__ void __launch_bounds__(256) append_kernel(DevState* st, uint4* kc, uint4* vc, uint4* ic,
                                                     const uint4* k, const uint4* v, const uint4* idx,
                                                     int n, int kv_units, int idx_units, int max_ctx,
                                                     float* kv_scales, int n_kv_heads, int hd) {
  pdl_launch_dependents();
  pdl_wait();
  const int base = ld_volatile(&st->n_ctx);
  const bool fits = base >= 0 && base + n <= max_ctx;
  if (fits) {
    const size_t nkv = size_t(n) * kv_units, nidx = size_t(n) * idx_units;
    const size_t okv = size_t(base) * kv_units, oidx = size_t(base) * idx_units;
    const size_t stride = size_t(gridDim.x) * blockDim.x;
    if constexpr (!FP8) {
      for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < nkv; i += stride) {
        kc[okv + i] = k[i];
        vc[okv + i] = v[i];
      }
    } else {
      const int lane = threadIdx.x & 31;
      const size_t rows = size_t(n) * n_kv_heads * 2, warps = stride / 32;
      for (size_t r = (size_t(blockIdx.x) * blockDim.x + threadIdx.x) / 32; r < rows; r += warps) {
        const size_t t = r / (2 * n_kv_heads);
        const KvRow kr = kv_row(int(r % (2 * n_kv_heads)), size_t(base) + t,
                                reinterpret_cast<const __half*>(k) + t * n_kv_heads * hd,
                                reinterpret_cast<const __half*>(v) + t * n_kv_heads * hd,
                                reinterpret_cast<unsigned char*>(kc), reinterpret_cast<unsigned char*>(vc), kv_scales,
                                n_kv_heads, hd);
        fp8_row_store(fp8_row_load(kr.src, hd, lane), kr.dst, kr.scale, hd, lane);
      }
    }
    for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < nidx; i += stride)
      ic[oidx + i] = idx[i];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned t = atomicAdd(&st->ticket_append, 1u);
    if (t == gridDim.x - 1) {
      if (fits) st->n_ctx = base + n;
      else record_status(st, QSA_ERR_CAPACITY);
      st->ticket_append = 0;
      __threadfence();
    }
  }
}

cudaError_t launch_append(const LayerView& L, int n, const void* k, const void* v, const void* idx,
                          int grid_hint, cudaStream_t s) {
  const int kv_units = L.cfg.n_kv_heads * L.cfg.head_dim * 2 / 16;
  const int idx_units = L.cfg.d_idx * 2 / 16;
  long long work = (long long)n * kv_units;
  int grid = int((work + 256 * 4 - 1) / (256 * 4));
  if (grid < 1) grid = 1;
  if (grid > grid_hint) grid = grid_hint;
  if (L.cfg.kv_format == QSA_KV_FP8)
    return launch_pdl(append_kernel<true>, dim3(grid), dim3(256), 0, s, 1, L.state, (uint4*)L.k_cache,
                      (uint4*)L.v_cache, (uint4*)L.idx_cache, (const uint4*)k, (const uint4*)v, (const uint4*)idx, n,
                      kv_units, idx_units, L.cfg.max_ctx, L.kv_scales, L.cfg.n_kv_heads, L.cfg.head_dim);
  return launch_pdl(append_kernel<false>, dim3(grid), dim3(256), 0, s, 1, L.state, (uint4*)L.k_cache,
                    (uint4*)L.v_cache, (uint4*)L.idx_cache, (const uint4*)k, (const uint4*)v, (const uint4*)idx, n,
                    kv_units, idx_units, L.cfg.max_ctx, L.kv_scales, L.cfg.n_kv_heads, L.cfg.head_dim);
}

constexpr int kPoolThreads = 256;

// Pools blocks [n_pooled, n_ctx/4), one warp per block, grid-stride.
template <int D, bool GEN>
__global__ void __launch_bounds__(kPoolThreads) pool_update_kernel(DevState* st, const __half* __restrict__ ic,
                                                                   PooledOut pc,
                                                                   const float* __restrict__ gain, float eps,
                                                                   PoolRope rope, int max_blocks) {
  __shared__ float s_rows[GEN ? kPoolThreads / 32 : 1][GEN ? D : 1];
  pdl_launch_dependents();
  pdl_wait();
  const int n = ld_volatile(&st->n_ctx);
  const int b_first = ld_volatile(&st->n_pooled);
  int b_end = n / kBlock;
  if (!QSA_GUARD(st, b_end <= max_blocks && b_first >= 0)) b_end = b_first;  // pool nothing
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const int gw = blockIdx.x * warps + (threadIdx.x >> 5);
  float* s_row = GEN ? s_rows[threadIdx.x >> 5] : nullptr;
  const PoolLane<D, GEN> c = pool_lane_consts<D, GEN>(lane, gain, rope.base, rope.dims, rope.interleaved);
  // warp gw takes blocks b_first + gw + u*W (W = all warps), kBatch of them per round with
  // every raw-key load of the round in flight before the first block is finished
  constexpr int kBatch = 4;
  const int W = gridDim.x * warps;
  for (int b0 = b_first + gw; b0 < b_end; b0 += kBatch * W) {
    PoolRaw<D> raw[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u)
      if (b0 + u * W < b_end) pool_load<D>(b0 + u * W, lane, ic, raw[u]);
#pragma unroll
    for (int u = 0; u < kBatch; ++u)
      if (b0 + u * W < b_end) pool_finish<D, GEN>(b0 + u * W, lane, c, raw[u], pc, eps, rope.pos, s_row);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned t = atomicAdd(&st->ticket_pool, 1u);
    if (t == gridDim.x - 1) {
      if (b_end > b_first) st->n_pooled = b_end;
      st->ticket_pool = 0;
      __threadfence();
    }
  }
}

// Decode-step append fused with the incremental pooled update: one CTA writes the token
// at position n_ctx, then pools every block in [n_pooled, (n_ctx+1)/4) (in decode: the
// block this token completes, every 4th step, or nothing). Same result as
// qsa_append_token followed by qsa_update_pooled_cache.
template <int D, bool GEN, bool FP8>
__global__ void __launch_bounds__(kPoolThreads) decode_append_kernel(DevState* st, uint4* kc, uint4* vc, uint4* ic,
                                                                     const uint4* k, const uint4* v,
                                                                     const uint4* idx, int kv_units, int max_ctx,
                                                                     PooledOut pc,
                                                                     const float* __restrict__ gain, float eps,
                                                                     PoolRope rope, float* kv_scales, int n_kv_heads,
                                                                     int hd) {
  constexpr int IDX_UNITS = D * 2 / 16;
  __shared__ float s_rows[GEN ? kPoolThreads / 32 : 1][GEN ? D : 1];
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  pdl_wait();
  // the token's first K/V/key units (FP8: each warp's first row), loaded in the same
  // round trip as the state
  const int t0 = threadIdx.x;
  uint4 k0 = make_uint4(0u, 0u, 0u, 0u), v0 = k0, i0 = k0;
  Fp8Row row0{};
  const __half* kh = reinterpret_cast<const __half*>(k);
  const __half* vh = reinterpret_cast<const __half*>(v);
  if constexpr (!FP8) {
    if (t0 < kv_units) {
      k0 = k[t0];
      v0 = v[t0];
    }
  } else {
    if (warp < 2 * n_kv_heads) row0 = fp8_row_load((warp & 1 ? vh : kh) + size_t(warp >> 1) * hd, hd, lane);
  }
  if (t0 < IDX_UNITS) i0 = idx[t0];
  const PoolLane<D, GEN> c = pool_lane_consts<D, GEN>(lane, gain, rope.base, rope.dims, rope.interleaved);
  const int n = ld_volatile(&st->n_ctx);
  const int b_first = ld_volatile(&st->n_pooled);
  asm volatile("" ::"r"(k0.x), "r"(k0.y), "r"(k0.z), "r"(k0.w), "r"(v0.x), "r"(v0.y), "r"(v0.z), "r"(v0.w));
  asm volatile("" ::"r"(i0.x), "r"(i0.y), "r"(i0.z), "r"(i0.w));
  asm volatile("" ::"f"(row0.x[0]), "f"(row0.x[1]), "f"(row0.x[2]), "f"(row0.x[3]));
  if (n < 0 || n >= max_ctx) {
    if (threadIdx.x == 0) record_status(st, QSA_ERR_CAPACITY);
    return;
  }
  if constexpr (!FP8) {
    if (t0 < kv_units) {
      kc[size_t(n) * kv_units + t0] = k0;
      vc[size_t(n) * kv_units + t0] = v0;
    }
    for (int i = t0 + blockDim.x; i < kv_units; i += blockDim.x) {  // heads beyond one pass
      kc[size_t(n) * kv_units + i] = k[i];
      vc[size_t(n) * kv_units + i] = v[i];
    }
  } else {
    unsigned char* kc8 = reinterpret_cast<unsigned char*>(kc);
    unsigned char* vc8 = reinterpret_cast<unsigned char*>(vc);
    const int warps = blockDim.x >> 5;
    for (int r = warp; r < 2 * n_kv_heads; r += warps) {
      const KvRow kr = kv_row(r, size_t(n), kh, vh, kc8, vc8, kv_scales, n_kv_heads, hd);
      fp8_row_store(r == warp ? row0 : fp8_row_load(kr.src, hd, lane), kr.dst, kr.scale, hd, lane);
    }
  }
  if (t0 < IDX_UNITS) ic[size_t(n) * IDX_UNITS + t0] = i0;
  __syncthreads();  // the new indexer key is visible to every warp of the CTA
  const int b_end = (n + 1) / kBlock;
  const __half* ich = reinterpret_cast<const __half*>(ic);
  float* s_row = GEN ? s_rows[warp] : nullptr;
  for (int b = b_first + warp; b < b_end; b += blockDim.x >> 5)
    pool_one_block<D, GEN>(b, lane, c, ich, pc, eps, rope.pos, s_row);
  __syncthreads();
  if (threadIdx.x == 0) {
    if (b_end > b_first) st->n_pooled = b_end;
    st->n_ctx = n + 1;
  }
}

namespace {
PoolRope pool_rope(const qsa_config& c) {
  return PoolRope{c.rope_base, c.rope_dims, c.rope_interleaved, RopePos{c.rope_pos_stride, c.rope_pos_offset}};
}
// Full-width NeoX pairs keep each rotation pair inside one lane (the common layout).
bool rope_generic(const qsa_config& c) { return c.rope_dims != c.d_idx || c.rope_interleaved != 0; }
}  // namespace

template <int D, bool GEN>
static cudaError_t launch_decode_append_d(const LayerView& L, const void* k, const void* v, const void* idx,
                                          cudaStream_t s) {
  const int kv_units = L.cfg.n_kv_heads * L.cfg.head_dim * 2 / 16;
#define QSA_DA_LAUNCH(F8)                                                                                         \
  launch_pdl(decode_append_kernel<D, GEN, F8>, dim3(1), dim3(kPoolThreads), 0, s, 1, L.state, (uint4*)L.k_cache,     \
             (uint4*)L.v_cache, (uint4*)L.idx_cache, (const uint4*)k, (const uint4*)v, (const uint4*)idx, kv_units, \
             L.cfg.max_ctx, pooled_out(L), L.rms_gain, L.cfg.rms_eps, pool_rope(L.cfg), L.kv_scales,    \
             L.cfg.n_kv_heads, L.cfg.head_dim)
  return L.cfg.kv_format == QSA_KV_FP8 ? QSA_DA_LAUNCH(true) : QSA_DA_LAUNCH(false);
#undef QSA_DA_LAUNCH
}

cudaError_t launch_decode_append(const LayerView& L, const void* k, const void* v, const void* idx, cudaStream_t s) {
  const bool gen = rope_generic(L.cfg);
  if (L.cfg.d_idx == 128)
    return gen ? launch_decode_append_d<128, true>(L, k, v, idx, s) : launch_decode_append_d<128, false>(L, k, v, idx, s);
  return gen ? launch_decode_append_d<64, true>(L, k, v, idx, s) : launch_decode_append_d<64, false>(L, k, v, idx, s);
}

template <int D, bool GEN>
static cudaError_t launch_pool_update_d(const LayerView& L, int grid, cudaStream_t s) {
  return launch_pdl(pool_update_kernel<D, GEN>, dim3(grid), dim3(kPoolThreads), 0, s, 1, L.state,
                    (const __half*)L.idx_cache, pooled_out(L), L.rms_gain, L.cfg.rms_eps, pool_rope(L.cfg),
                    L.cfg.max_ctx / kBlock);
}

cudaError_t launch_pool_update(const LayerView& L, int grid_hint, cudaStream_t s) {
  const int grid = grid_hint < 1 ? 1 : grid_hint;
  const bool gen = rope_generic(L.cfg);
  if (L.cfg.d_idx == 128)
    return gen ? launch_pool_update_d<128, true>(L, grid, s) : launch_pool_update_d<128, false>(L, grid, s);
  return gen ? launch_pool_update_d<64, true>(L, grid, s) : launch_pool_update_d<64, false>(L, grid, s);
}

}  // namespace qsa
