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

#include "qsa_device.cuh"
#include "qsa_checked.cuh"

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

// FP8 K/V rows (an 8-bit K/V cache, as tried in the Qwen3.8-Flash-Next parameter-tuning
// post on EVO-X2, section "KV cacheをQ8_0にしてみる"; here in e4m3 form): one warp quantises
// one (token, KV head) row of hd = 64 or 128 f16 values, E = hd/32 per lane:
// scale = amax/448, codes = e4m3(x * (448/amax)) rounded to nearest-even and saturated
// (an all-zero row: scale 1, zero codes). The scale and the multiplier are single f32
// divisions and each code one f32 product, so the codes are exactly reproducible.
struct Fp8Row {
  float x[4];
};

__device__ __forceinline__ Fp8Row fp8_row_load(const __half* src, int hd, int lane) {
  Fp8Row r;
  if (hd == 128) {
    const uint2 u = *reinterpret_cast<const uint2*>(src + lane * 4);
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
    r.x[0] = a.x, r.x[1] = a.y, r.x[2] = b.x, r.x[3] = b.y;
  } else {
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(src + lane * 2));
    r.x[0] = a.x, r.x[1] = a.y, r.x[2] = 0.0f, r.x[3] = 0.0f;
  }
  return r;
}

__device__ __forceinline__ void fp8_row_store(const Fp8Row& r, unsigned char* dst, float* scale_dst, int hd,
                                              int lane) {
  float m = fmaxf(fmaxf(fabsf(r.x[0]), fabsf(r.x[1])), fmaxf(fabsf(r.x[2]), fabsf(r.x[3])));
  m = warp_max(m);
  const float scale = m > 0.0f ? m / 448.0f : 1.0f;
  const float mult = m > 0.0f ? 448.0f / m : 0.0f;
  const uint32_t p0 = __nv_cvt_float2_to_fp8x2(make_float2(__fmul_rn(r.x[0], mult), __fmul_rn(r.x[1], mult)),
                                               __NV_SATFINITE, __NV_E4M3);
  if (hd == 128) {
    const uint32_t p1 = __nv_cvt_float2_to_fp8x2(make_float2(__fmul_rn(r.x[2], mult), __fmul_rn(r.x[3], mult)),
                                                 __NV_SATFINITE, __NV_E4M3);
    *reinterpret_cast<uint32_t*>(dst + lane * 4) = p0 | (p1 << 16);
  } else {
    *reinterpret_cast<uint16_t*>(dst + lane * 2) = uint16_t(p0);
  }
  if (lane == 0) *scale_dst = scale;
}

// Row r of a token's K/V (r < 2*Hkv: head r/2, K when r is even, V when odd).
struct KvRow {
  const __half* src;
  unsigned char* dst;
  float* scale;
};

__device__ __forceinline__ KvRow kv_row(int r, size_t token, const __half* k, const __half* v, unsigned char* kc8,
                                        unsigned char* vc8, float* kv_scales, int n_kv_heads, int hd) {
  const int h = r >> 1, is_v = r & 1;
  const size_t row = token * n_kv_heads + h;
  return KvRow{(is_v ? v : k) + size_t(h) * hd, (is_v ? vc8 : kc8) + row * hd, kv_scales + row * 2 + is_v};
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

// Summary of block b computed by one warp. Lane `lane` owns the elements i = lane*P + j
// (j < P, P = D/64) and i + D/2. In the default layout (all D dims rotary, NeoX pairs)
// those are exactly the lane's rotation pairs; GEN kernels handle partial rotary and
// interleaved pairs, whose partners may sit in other lanes, through a per-warp row of
// shared memory. theta/g1/g2 are the lane's RoPE frequencies and gains.
template <int D, bool GEN>
struct PoolLane {  // default layout: pair j of the lane is (lane*P + j, lane*P + j + D/2)
  static constexpr int P = D / 64;
  double theta[P];
  float g1[P], g2[P];
};

template <int D>
struct PoolLane<D, true> {  // slot k < P is element lane*P + k, slot P + j is lane*P + j + D/2
  static constexpr int P = D / 64;
  double theta[2 * P];
  float g1[P], g2[P];
  int partner[2 * P];
  float sign[2 * P];
};

template <int D, bool GEN>
__device__ __forceinline__ int pool_elem(int lane, int k) {
  constexpr int P = PoolLane<D, GEN>::P;
  return k < P ? lane * P + k : lane * P + (k - P) + D / 2;
}

template <int D, bool GEN>
__device__ __forceinline__ PoolLane<D, GEN> pool_lane_consts(int lane, const float* __restrict__ gain,
                                                             float rope_base, int rope_dims, int interleaved) {
  PoolLane<D, GEN> c;
  constexpr int P = PoolLane<D, GEN>::P;
#pragma unroll
  for (int j = 0; j < P; ++j) {
    const int i = lane * P + j;
    c.g1[j] = gain ? gain[i] : 1.0f;
    c.g2[j] = gain ? gain[i + D / 2] : 1.0f;
    if constexpr (!GEN) c.theta[j] = pow((double)rope_base, -2.0 * (double)i / (double)D);
  }
  if constexpr (GEN) {
#pragma unroll
    for (int k = 0; k < 2 * P; ++k) {
      const RopeSlot r = rope_slot(pool_elem<D, GEN>(lane, k), rope_dims, interleaved != 0);
      c.partner[k] = r.partner;
      c.sign[k] = r.sign;
      c.theta[k] = r.freq < 0 ? 0.0 : pow((double)rope_base, -2.0 * (double)r.freq / (double)rope_dims);
    }
  }
  return c;
}

// cos and sin of the RoPE angle pos * theta. The angle is formed and reduced modulo 2*pi
// in double (|angle| <= ~4.2e6 rad: the reduced angle is exact to ~1e-9 rad), then
// evaluated with the hardware approximation, whose absolute error on [-pi, pi] is below
// 4e-7, three orders below the f16 rounding of the pooled row. The positions reach 2^18
// and more, where a float angle would already be off by ~0.016 rad; the reduction in
// double avoids that. Decode and bulk pooling share this routine, so they stay
// bit-identical.
__device__ __forceinline__ void rope_cos_sin(double pos, double theta, float* cs, float* sn) {
  constexpr double kTwoPi = 6.283185307179586;
  const double angle = pos * theta;
  const double r = fma(-rint(angle * (1.0 / kTwoPi)), kTwoPi, angle);
  __sincosf(float(r), sn, cs);
}

// Where a block sits on the RoPE position scale: stride*b + offset (4b by default).
struct RopePos {
  int stride, offset;
};

// The 4 raw indexer keys of one block as one lane of a warp holds them (f16, packed):
// elements i = lane*P + j (j < P) and i + D/2.
template <int D>
struct PoolRaw {
  __half2 x1[kBlock], x2[kBlock];  // P == 1 uses the low half only
};

// `ic` is deliberately not __restrict__: the fused decode kernel reads back a row it has
// just written, which must not go through the non-coherent load path.
template <int D>
__device__ __forceinline__ void pool_load(int b, int lane, const __half* ic, PoolRaw<D>& raw) {
  constexpr int P = D / 64;
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
// the block position, f16 store. GEN kernels pass s_row, D floats of shared memory owned
// by the warp.
template <int D, bool GEN>
__device__ __forceinline__ void pool_finish(int b, int lane, const PoolLane<D, GEN>& c, const PoolRaw<D>& raw,
                                            __half* __restrict__ pc, float eps, RopePos rp, float* s_row) {
  constexpr int P = D / 64;
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
  const double pos = (double)(rp.stride * b + rp.offset);
  __half o1[P], o2[P];
  if constexpr (!GEN) {
#pragma unroll
    for (int j = 0; j < P; ++j) {
      const float r1 = m1[j] * inv_rms * c.g1[j];
      const float r2 = m2[j] * inv_rms * c.g2[j];
      float cs, sn;
      rope_cos_sin(pos, c.theta[j], &cs, &sn);
      o1[j] = __float2half_rn(r1 * cs - r2 * sn);
      o2[j] = __float2half_rn(r1 * sn + r2 * cs);
    }
  } else {
    float r[2 * P];
#pragma unroll
    for (int j = 0; j < P; ++j) {
      r[j] = m1[j] * inv_rms * c.g1[j];
      r[P + j] = m2[j] * inv_rms * c.g2[j];
    }
#pragma unroll
    for (int k = 0; k < 2 * P; ++k) s_row[pool_elem<D, GEN>(lane, k)] = r[k];
    __syncwarp();
    float o[2 * P];
#pragma unroll
    for (int k = 0; k < 2 * P; ++k) {
      o[k] = r[k];
      if (c.sign[k] != 0.0f) {
        float cs, sn;
        rope_cos_sin(pos, c.theta[k], &cs, &sn);
        o[k] = r[k] * cs + c.sign[k] * s_row[c.partner[k]] * sn;
      }
    }
    __syncwarp();  // the row is read before the warp's next block overwrites it
#pragma unroll
    for (int j = 0; j < P; ++j) {
      o1[j] = __float2half_rn(o[j]);
      o2[j] = __float2half_rn(o[P + j]);
    }
  }
  if constexpr (P == 2) {
    *reinterpret_cast<__half2*>(pc + size_t(b) * D + lane * 2) = __halves2half2(o1[0], o1[1]);
    *reinterpret_cast<__half2*>(pc + size_t(b) * D + lane * 2 + HALF) = __halves2half2(o2[0], o2[1]);
  } else {
    pc[size_t(b) * D + lane] = o1[0];
    pc[size_t(b) * D + lane + HALF] = o2[0];
  }
}

template <int D, bool GEN>
__device__ __forceinline__ void pool_one_block(int b, int lane, const PoolLane<D, GEN>& c, const __half* ic,
                                               __half* __restrict__ pc, float eps, RopePos rp, float* s_row) {
  PoolRaw<D> raw;
  pool_load<D>(b, lane, ic, raw);
  pool_finish<D, GEN>(b, lane, c, raw, pc, eps, rp, s_row);
}

// RoPE settings of a layer as the pooling kernels take them.
struct PoolRope {
  float base;
  int dims, interleaved;
  RopePos pos;
};

constexpr int kPoolThreads = 256;

// Pools blocks [n_pooled, n_ctx/4), one warp per block, grid-stride.
template <int D, bool GEN>
__global__ void __launch_bounds__(kPoolThreads) pool_update_kernel(DevState* st, const __half* __restrict__ ic,
                                                                   __half* __restrict__ pc,
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
                                                                     __half* __restrict__ pc,
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
             L.cfg.max_ctx, (__half*)L.pooled_cache, L.rms_gain, L.cfg.rms_eps, pool_rope(L.cfg), L.kv_scales,    \
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
                    (const __half*)L.idx_cache, (__half*)L.pooled_cache, L.rms_gain, L.cfg.rms_eps, pool_rope(L.cfg),
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
