// Device routines of the pooled-key summary and of the FP8 K/V row format, shared by the
// cache kernels (qsa_cache.cu) and the decode-step scan that appends and pools in its
// own prologue (qsa_scan_tc.cu).
//
// Incremental pooled-key cache: web page "Part 10" (第10回 EVO-X2 ... 長コンテキストのTGを
// 高速化した話), section "incremental pooled-key cache（COMMON-004）"; summary of block b
// (section "QSA indexer"): mean of its 4 raw indexer keys -> RMS norm -> RoPE at the
// block position, stored as f16.
#pragma once

#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "qsa_device.cuh"

namespace qsa {

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

// Where a summary goes: the f16 pooled cache, or with 8-bit pooled keys (scale != null)
// its e4m3 codes and the row's scale.
struct PooledOut {
  __half* f16;
  unsigned char* fp8;
  float* scale;
};

// The layer's pooled cache in the form its pooled_format stores.
inline PooledOut pooled_out(const LayerView& L) {
  const bool fp8 = L.cfg.pooled_format == QSA_POOLED_FP8;
  return PooledOut{fp8 ? nullptr : static_cast<__half*>(L.pooled_cache),
                   fp8 ? static_cast<unsigned char*>(L.pooled_cache) : nullptr, fp8 ? L.pooled_scales : nullptr};
}

// Summary of block b from its raw keys: mean (summed in token order), RMSNorm, RoPE at
// the block position, f16 store (or the f16 row quantised to e4m3 codes and one scale by
// the FP8 K/V rule, for 8-bit pooled keys). GEN kernels pass s_row, D floats of shared
// memory owned by the warp.
template <int D, bool GEN>
__device__ __forceinline__ void pool_finish(int b, int lane, const PoolLane<D, GEN>& c, const PoolRaw<D>& raw,
                                            const PooledOut& out, float eps, RopePos rp, float* s_row) {
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
    if (out.scale) {  // 8-bit pooled keys (d_idx 128): scale = amax/448, codes of x * 448/amax
      const float x0 = __half2float(o1[0]), x1 = __half2float(o1[1]);
      const float x2 = __half2float(o2[0]), x3 = __half2float(o2[1]);
      const float m = warp_max(fmaxf(fmaxf(fabsf(x0), fabsf(x1)), fmaxf(fabsf(x2), fabsf(x3))));
      const float scale = m > 0.0f ? m / 448.0f : 1.0f;
      const float mult = m > 0.0f ? 448.0f / m : 0.0f;
      const uint32_t p0 = __nv_cvt_float2_to_fp8x2(make_float2(__fmul_rn(x0, mult), __fmul_rn(x1, mult)),
                                                   __NV_SATFINITE, __NV_E4M3);
      const uint32_t p1 = __nv_cvt_float2_to_fp8x2(make_float2(__fmul_rn(x2, mult), __fmul_rn(x3, mult)),
                                                   __NV_SATFINITE, __NV_E4M3);
      unsigned char* row = out.fp8 + size_t(b) * D;
      *reinterpret_cast<uint16_t*>(row + lane * 2) = uint16_t(p0);
      *reinterpret_cast<uint16_t*>(row + lane * 2 + HALF) = uint16_t(p1);
      if (lane == 0) out.scale[b] = scale;
      return;
    }
    *reinterpret_cast<__half2*>(out.f16 + size_t(b) * D + lane * 2) = __halves2half2(o1[0], o1[1]);
    *reinterpret_cast<__half2*>(out.f16 + size_t(b) * D + lane * 2 + HALF) = __halves2half2(o2[0], o2[1]);
  } else {
    out.f16[size_t(b) * D + lane] = o1[0];
    out.f16[size_t(b) * D + lane + HALF] = o2[0];
  }
}

template <int D, bool GEN>
__device__ __forceinline__ void pool_one_block(int b, int lane, const PoolLane<D, GEN>& c, const __half* ic,
                                               const PooledOut& out, float eps, RopePos rp, float* s_row) {
  PoolRaw<D> raw;
  pool_load<D>(b, lane, ic, raw);
  pool_finish<D, GEN>(b, lane, c, raw, out, eps, rp, s_row);
}

// RoPE settings of a layer as the pooling kernels take them.
struct PoolRope {
  float base;
  int dims, interleaved;
  RopePos pos;
};

}  // namespace qsa
