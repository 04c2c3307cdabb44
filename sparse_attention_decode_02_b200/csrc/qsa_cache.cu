// Sequence state, token append and the incremental pooled-key cache.
//
// Incremental pooled-key cache: web page "Part 10" (第10回 EVO-X2 ... 長コンテキストのTGを
// 高速化した話), section "incremental pooled-key cache（COMMON-004）": completed-block
// summaries are kept per layer and only blocks that completed (or were invalidated)
// since the last update are computed. Summary of block b (section "QSA indexer"):
// mean of its 4 raw indexer keys -> RMS norm -> RoPE at the block position 4b, stored
// as f16. RoPE is the NeoX half-split rotation of pair (i, i+d/2) by angle
// pos * base^(-2i/d); angles and their sine/cosine are taken in double precision so that
// positions near 2.6e5 keep full accuracy, then the rotation itself runs in f32.
#include <cuda_fp16.h>

#include "qsa_device.cuh"

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
  } else {
    st->status = 0;
  }
}

cudaError_t launch_set_state(const LayerView& L, int n_ctx, int n_pooled, int mode, cudaStream_t s) {
  return launch_pdl(set_state_kernel, dim3(1), dim3(32), 0, s, 1, L.state, n_ctx, n_pooled, mode);
}

// Appends n tokens at position n_ctx: three contiguous copies (token-major caches), in
// 16-byte units. All CTAs read n_ctx before any of them can change it: the last CTA to
// finish (atomic ticket) publishes n_ctx + n.
__global__ void __launch_bounds__(256) append_kernel(DevState* st, uint4* kc, uint4* vc, uint4* ic,
                                                     const uint4* k, const uint4* v, const uint4* idx,
                                                     int n, int kv_units, int idx_units, int max_ctx) {
  pdl_launch_dependents();
  pdl_wait();
  const int base = ld_volatile(&st->n_ctx);
  const bool fits = base >= 0 && base + n <= max_ctx;
  if (fits) {
    const size_t nkv = size_t(n) * kv_units, nidx = size_t(n) * idx_units;
    const size_t okv = size_t(base) * kv_units, oidx = size_t(base) * idx_units;
    const size_t stride = size_t(gridDim.x) * blockDim.x;
    for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < nkv; i += stride) {
      kc[okv + i] = k[i];
      vc[okv + i] = v[i];
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
  return launch_pdl(append_kernel, dim3(grid), dim3(256), 0, s, 1, L.state, (uint4*)L.k_cache,
                    (uint4*)L.v_cache, (uint4*)L.idx_cache, (const uint4*)k, (const uint4*)v,
                    (const uint4*)idx, n, kv_units, idx_units, L.cfg.max_ctx);
}

// Summary of block b computed by one warp. Lane `lane` owns the rotation pairs
// i = lane*P + j (j < P, P = D/64) and their partners i + D/2. theta/g1/g2 are the
// lane's RoPE frequencies and gains (see pool_lane_consts).
template <int D>
struct PoolLane {
  static constexpr int P = D / 64;
  double theta[P];
  float g1[P], g2[P];
};

template <int D>
__device__ __forceinline__ PoolLane<D> pool_lane_consts(int lane, const float* __restrict__ gain, float rope_base) {
  PoolLane<D> c;
#pragma unroll
  for (int j = 0; j < PoolLane<D>::P; ++j) {
    const int i = lane * PoolLane<D>::P + j;
    c.theta[j] = pow((double)rope_base, -2.0 * (double)i / (double)D);
    c.g1[j] = gain ? gain[i] : 1.0f;
    c.g2[j] = gain ? gain[i + D / 2] : 1.0f;
  }
  return c;
}

// cos and sin of the RoPE angle pos * theta. The angle is formed and reduced modulo 2*pi
// in double (|angle| <= ~2.6e5 rad: the reduced angle is exact to ~1e-11 rad), then
// evaluated with the hardware approximation, whose absolute error on [-pi, pi] is below
// 4e-7, three orders below the f16 rounding of the pooled row. The positions reach 2^18,
// where a float angle would already be off by ~0.016 rad; the reduction in double avoids
// that. Decode and bulk pooling share this routine, so they stay bit-identical.
__device__ __forceinline__ void rope_cos_sin(double pos, double theta, float* cs, float* sn) {
  constexpr double kTwoPi = 6.283185307179586;
  const double angle = pos * theta;
  const double r = fma(-rint(angle * (1.0 / kTwoPi)), kTwoPi, angle);
  __sincosf(float(r), sn, cs);
}

// The 4 raw indexer keys of one block as one lane of a warp holds them (f16, packed):
// rotation pairs i = lane*P + j (j < P) and their partners i + D/2.
template <int D>
struct PoolRaw {
  __half2 x1[kBlock], x2[kBlock];  // P == 1 uses the low half only
};

// `ic` is deliberately not __restrict__: the fused decode kernel reads back a row it has
// just written, which must not go through the non-coherent load path.
template <int D>
__device__ __forceinline__ void pool_load(int b, int lane, const __half* ic, PoolRaw<D>& raw) {
  constexpr int P = PoolLane<D>::P;
  constexpr int HALF = D / 2;
  static_assert(P == 1 || P == 2, "one or two rotation pairs per lane");
#pragma unroll
  for (int t = 0; t < kBlock; ++t) {
    const __half* row = ic + (size_t(b) * kBlock + t) * D;
    if constexpr (P == 2) {
      raw.x1[t] = *reinterpret_cast<const __half2*>(row + lane * 2);
      raw.x2[t] = *reinterpret_cast<const __half2*>(row + lane * 2 + HALF);
    } else {
      raw.x1[t] = __halves2half2(row[lane], __float2half_rn(0.0f));
      raw.x2[t] = __halves2half2(row[lane + HALF], __float2half_rn(0.0f));
    }
  }
}

// Summary of block b from its raw keys: mean (summed in token order), RMSNorm, RoPE at
// the block position 4b, f16 store.
template <int D>
__device__ __forceinline__ void pool_finish(int b, int lane, const PoolLane<D>& c, const PoolRaw<D>& raw,
                                            __half* __restrict__ pc, float eps) {
  constexpr int P = PoolLane<D>::P;
  constexpr int HALF = D / 2;
  float m1[P], m2[P];
#pragma unroll
  for (int j = 0; j < P; ++j) m1[j] = m2[j] = 0.0f;
#pragma unroll
  for (int t = 0; t < kBlock; ++t) {
    const float2 a = __half22float2(raw.x1[t]), z = __half22float2(raw.x2[t]);
    m1[0] += a.x;
    m2[0] += z.x;
    if constexpr (P == 2) {
      m1[P - 1] += a.y;
      m2[P - 1] += z.y;
    }
  }
  float ss = 0.0f;
#pragma unroll
  for (int j = 0; j < P; ++j) {
    m1[j] *= 0.25f;
    m2[j] *= 0.25f;
    ss += m1[j] * m1[j] + m2[j] * m2[j];
  }
  ss = warp_sum(ss);
  const float inv_rms = 1.0f / sqrtf(ss / (float)D + eps);
  const double pos = (double)(b * kBlock);
  __half o1[P], o2[P];
#pragma unroll
  for (int j = 0; j < P; ++j) {
    const float r1 = m1[j] * inv_rms * c.g1[j];
    const float r2 = m2[j] * inv_rms * c.g2[j];
    float cs, sn;
    rope_cos_sin(pos, c.theta[j], &cs, &sn);
    o1[j] = __float2half_rn(r1 * cs - r2 * sn);
    o2[j] = __float2half_rn(r1 * sn + r2 * cs);
  }
  if constexpr (P == 2) {
    *reinterpret_cast<__half2*>(pc + size_t(b) * D + lane * 2) = __halves2half2(o1[0], o1[1]);
    *reinterpret_cast<__half2*>(pc + size_t(b) * D + lane * 2 + HALF) = __halves2half2(o2[0], o2[1]);
  } else {
    pc[size_t(b) * D + lane] = o1[0];
    pc[size_t(b) * D + lane + HALF] = o2[0];
  }
}

template <int D>
__device__ __forceinline__ void pool_one_block(int b, int lane, const PoolLane<D>& c, const __half* ic,
                                               __half* __restrict__ pc, float eps) {
  PoolRaw<D> raw;
  pool_load<D>(b, lane, ic, raw);
  pool_finish<D>(b, lane, c, raw, pc, eps);
}

// Pools blocks [n_pooled, n_ctx/4), one warp per block, grid-stride.
template <int D>
__global__ void __launch_bounds__(256) pool_update_kernel(DevState* st, const __half* __restrict__ ic,
                                                          __half* __restrict__ pc,
                                                          const float* __restrict__ gain, float eps,
                                                          float rope_base) {
  pdl_launch_dependents();
  pdl_wait();
  const int n = ld_volatile(&st->n_ctx);
  const int b_first = ld_volatile(&st->n_pooled);
  const int b_end = n / kBlock;
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const int gw = blockIdx.x * warps + (threadIdx.x >> 5);
  const PoolLane<D> c = pool_lane_consts<D>(lane, gain, rope_base);
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
      if (b0 + u * W < b_end) pool_finish<D>(b0 + u * W, lane, c, raw[u], pc, eps);
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
template <int D>
__global__ void __launch_bounds__(256) decode_append_kernel(DevState* st, uint4* kc, uint4* vc, uint4* ic,
                                                            const uint4* k, const uint4* v, const uint4* idx,
                                                            int kv_units, int max_ctx, __half* __restrict__ pc,
                                                            const float* __restrict__ gain, float eps,
                                                            float rope_base) {
  constexpr int IDX_UNITS = D * 2 / 16;
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  pdl_wait();
  // the token's first K/V/key units, loaded in the same round trip as the state
  const int t0 = threadIdx.x;
  uint4 k0 = make_uint4(0u, 0u, 0u, 0u), v0 = k0, i0 = k0;
  if (t0 < kv_units) {
    k0 = k[t0];
    v0 = v[t0];
  }
  if (t0 < IDX_UNITS) i0 = idx[t0];
  const PoolLane<D> c = pool_lane_consts<D>(lane, gain, rope_base);
  const int n = ld_volatile(&st->n_ctx);
  const int b_first = ld_volatile(&st->n_pooled);
  asm volatile("" ::"r"(k0.x), "r"(k0.y), "r"(k0.z), "r"(k0.w), "r"(v0.x), "r"(v0.y), "r"(v0.z), "r"(v0.w));
  asm volatile("" ::"r"(i0.x), "r"(i0.y), "r"(i0.z), "r"(i0.w));
  if (n < 0 || n >= max_ctx) {
    if (threadIdx.x == 0) record_status(st, QSA_ERR_CAPACITY);
    return;
  }
  if (t0 < kv_units) {
    kc[size_t(n) * kv_units + t0] = k0;
    vc[size_t(n) * kv_units + t0] = v0;
  }
  for (int i = t0 + blockDim.x; i < kv_units; i += blockDim.x) {  // heads beyond one pass
    kc[size_t(n) * kv_units + i] = k[i];
    vc[size_t(n) * kv_units + i] = v[i];
  }
  if (t0 < IDX_UNITS) ic[size_t(n) * IDX_UNITS + t0] = i0;
  __syncthreads();  // the new indexer key is visible to every warp of the CTA
  const int b_end = (n + 1) / kBlock;
  const __half* ich = reinterpret_cast<const __half*>(ic);
  for (int b = b_first + warp; b < b_end; b += blockDim.x >> 5) pool_one_block<D>(b, lane, c, ich, pc, eps);
  __syncthreads();
  if (threadIdx.x == 0) {
    if (b_end > b_first) st->n_pooled = b_end;
    st->n_ctx = n + 1;
  }
}

cudaError_t launch_decode_append(const LayerView& L, const void* k, const void* v, const void* idx, cudaStream_t s) {
  const int kv_units = L.cfg.n_kv_heads * L.cfg.head_dim * 2 / 16;
  if (L.cfg.d_idx == 128)
    return launch_pdl(decode_append_kernel<128>, dim3(1), dim3(256), 0, s, 1, L.state, (uint4*)L.k_cache,
                      (uint4*)L.v_cache, (uint4*)L.idx_cache, (const uint4*)k, (const uint4*)v, (const uint4*)idx,
                      kv_units, L.cfg.max_ctx, (__half*)L.pooled_cache, L.rms_gain, L.cfg.rms_eps,
                      L.cfg.rope_base);
  return launch_pdl(decode_append_kernel<64>, dim3(1), dim3(256), 0, s, 1, L.state, (uint4*)L.k_cache,
                    (uint4*)L.v_cache, (uint4*)L.idx_cache, (const uint4*)k, (const uint4*)v, (const uint4*)idx,
                    kv_units, L.cfg.max_ctx, (__half*)L.pooled_cache, L.rms_gain, L.cfg.rms_eps, L.cfg.rope_base);
}

cudaError_t launch_pool_update(const LayerView& L, int grid_hint, cudaStream_t s) {
  const int grid = grid_hint < 1 ? 1 : grid_hint;
  if (L.cfg.d_idx == 128)
    return launch_pdl(pool_update_kernel<128>, dim3(grid), dim3(256), 0, s, 1, L.state,
                      (const __half*)L.idx_cache, (__half*)L.pooled_cache, L.rms_gain, L.cfg.rms_eps,
                      L.cfg.rope_base);
  return launch_pdl(pool_update_kernel<64>, dim3(grid), dim3(256), 0, s, 1, L.state,
                    (const __half*)L.idx_cache, (__half*)L.pooled_cache, L.rms_gain, L.cfg.rms_eps,
                    L.cfg.rope_base);
}

}  // namespace qsa
