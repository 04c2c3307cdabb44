// Indexer scan on the 5th-generation tensor cores (tcgen05) with TMA streaming.
//
// Web page "Part 10" (第10回 EVO-X2 ... 長コンテキストのTGを高速化した話), section
// "QSA indexer": the current indexer query is scored against every completed block's
// pooled summary. This library's score (the pages give no formula):
//    score_b = sum_h w_h * max(0, q~_h . p_b) / sqrt(d),   q~_h = RoPE(q_h, n-1)
// (the query's RoPE follows the layer's rotary settings, like the pooled keys).
//
// The dots q~_h . p_b for all B blocks and H heads form a dense [B x d] . [d x H]
// contraction over f16 pooled rows, which at d = 128, H = 16 needs 8 FMA per byte read:
// more than the CUDA cores sustain at HBM rate, so it runs on the tensor cores:
//  - the rotated f32 query is split into two f16 matrices, q~ = hi + lo * 2^-12
//    (hi = f16(q~), lo = f16((q~ - hi) * 2^12)); both are the B operand (N = 2H columns,
//    padded to 16), so one MMA pass yields hi and lo dots accumulated in f32 and the
//    epilogue adds them: the query keeps ~22 significant bits instead of f16's 11;
//  - each CTA (one per SM) owns a contiguous range of pooled rows; warp 4 streams them
//    with TMA (16-row boxes, 128-byte swizzle) into a 6-stage shared-memory ring,
//    warp 5 issues tcgen05.mma (M = 128 rows) into one of 4 TMEM accumulators, and
//    warps 0-3 read the accumulator back (one row per thread) and form the score.
// No tile is re-read: every pooled byte crosses HBM once (plus at most 15 rows per CTA
// of rounding to the 16-row box).
//
// Two options ride on the same kernel:
//  - HIST: the epilogue also counts every score's 11-bit key prefix (the sign, exponent
//    and two mantissa bits of the order-preserving key the selection ranks by) into a
//    2048-bin histogram in the layer workspace, so the selection kernel starts from the
//    bin that holds the K-th score instead of running its own first radix pass;
//  - FUSED (the decode step): the kernel first appends the token (K/V row and indexer key
//    at position n_ctx) and, when that token completes a block, pools the block (section
//    "incremental pooled-key cache（COMMON-004）": only the new block is computed) before
//    scoring it, so a decode step needs no separate append launch. A seventh warp of the
//    CTA that owns the last rows does both; the new pooled row reaches the TMA loads
//    through a proxy fence and an mbarrier. The state is left for the selection kernel
//    that follows to advance (it counts the appended token), so the CTAs leave without a
//    ticket round trip.
#include <cuda.h>
#include <cuda_fp16.h>

#include "qsa_device.cuh"
#include "qsa_pool.cuh"
#include "qsa_select.cuh"
#include "qsa_sm100.cuh"
#include "qsa_timeline.cuh"

namespace qsa {

namespace {

using namespace sm100;

constexpr int kBoxRows = 16;     // TMA box height
constexpr int kF8Terms = 5;      // e4m3 terms of the query with 8-bit pooled keys (4 bits each)
// warps 0-3 epilogue, warp 4 TMA, warp 5 MMA + TMEM owner, warp 6 append + pool (FUSED)
constexpr int kThreads = 224;
constexpr float kLoScale = 4096.0f;
constexpr int kHistBins = 1 << kHistBits;

constexpr size_t kSmemMax = 227 * 1024;  // dynamic shared memory per CTA
#ifndef QSA_SCAN_STAGES
#define QSA_SCAN_STAGES 3
#endif
constexpr int kScanStages = QSA_SCAN_STAGES;  // TMA ring depth (tiles of 128 rows)

// Shapes of the scan for d = D, H indexer heads and T queries scored in one pass; F8:
// 8-bit pooled keys (e4m3 rows, the query as kF8Terms e4m3 terms).
template <int D, int H, int T, bool F8 = false>
struct ScanShape {
  static constexpr int ESIZE = F8 ? 1 : 2;                // bytes per pooled element
  static constexpr int HALVES = D * ESIZE / 128;          // 128-byte swizzle spans per row
  static constexpr int TERMS = F8 ? kF8Terms : 2;        // query terms: hi and lo, or e4m3 terms
  static constexpr int NQ = (TERMS * H + 15) / 16 * 16;  // B rows per query (term-major), zero pad
  static constexpr int N = T * NQ;                        // MMA N
  static constexpr int K_STEPS = D * ESIZE / 32;          // MMAs per tile: 32 bytes of K each
  static constexpr int ACC = F8 ? 2 : 4;                  // TMEM accumulators
  static constexpr int TILE_BYTES = 128 * D * ESIZE;      // A tile: 128 rows
  static constexpr int HALF_BYTES = 128 * 128;            // 128 rows x 128 bytes
  static constexpr int B_HALF_BYTES = N * 128;
  static constexpr int B_BYTES = N * D * ESIZE;
  static constexpr int ACC_COLS = ACC * N;
  static constexpr int TMEM_COLS =
      ACC_COLS <= 32 ? 32 : ACC_COLS <= 64 ? 64 : ACC_COLS <= 128 ? 128 : ACC_COLS <= 256 ? 256 : 512;
  static constexpr uint32_t IDESC = idesc_f16_f32(128, N);
  // barriers and TMEM address (256 B), sin/cos (T*D floats), RoPE frequencies (D/2
  // doubles), raw queries (T*H*D f16), the score-prefix histogram, one pooled row (f32),
  // the rotated query in f32 (8-bit keys: T*H*D floats)
  static constexpr int CTRL_BYTES =
      256 + T * D * 4 + D / 2 * 8 + T * H * D * 2 + T * kHistBins * 4 + D * 4 + (F8 ? T * H * D * 4 : 0);
  static constexpr size_t FIXED = 1024 + size_t(B_BYTES) + CTRL_BYTES;
  // ring depth: kScanStages tiles where they fit, fewer for wide B operands. A short ring
  // keeps the CTA small enough to be resident beside the attention and selection kernels'
  // CTAs, so it can start (and prefetch) while they still run.
  static constexpr int STAGES = FIXED + kScanStages * size_t(TILE_BYTES) <= kSmemMax ? kScanStages
                                : FIXED + 5 * size_t(TILE_BYTES) <= kSmemMax ? 5 : 4;
  static constexpr size_t SMEM = FIXED + size_t(STAGES) * TILE_BYTES;
  static_assert(NQ <= 80 && NQ % 16 == 0, "the epilogue reads the query's columns 16 at a time");
  static_assert(!F8 || (T == 1 && D == 128), "8-bit pooled keys: one query, d_idx 128");
  static_assert(N <= 256 && ACC_COLS <= 512, "MMA N and TMEM columns");
  static_assert(SMEM <= kSmemMax, "shared memory");
  static_assert(TILE_BYTES % 1024 == 0 && B_HALF_BYTES % 1024 == 0, "1024-byte swizzle atoms");
};

// Byte offset of element (row n, column k) of a K-major operand in the 128-byte swizzle
// layout (the layout TMA's SWIZZLE_128B writes): 64-column halves of `half_bytes` each,
// 8-row atoms of 1024 bytes, 16-byte chunk index XOR (row % 8).
__device__ __forceinline__ uint32_t sw128_offset(int n, int k, int half_bytes) {
  const int j = k >> 6, c = k & 63;
  return uint32_t(j * half_bytes + (n >> 3) * 1024 + (n & 7) * 128 + (((c >> 3) ^ (n & 7)) << 4) + ((c & 7) << 1));
}

// The same for a one-byte element at column k < 128 (one 128-byte span).
__device__ __forceinline__ uint32_t sw128_offset_b(int n, int k) {
  return uint32_t((n >> 3) * 1024 + (n & 7) * 128 + (((k >> 4) ^ (n & 7)) << 4) + (k & 15));
}

// D[tmem] (+)= A[smem] * B[smem]^T with e4m3 operands (kind::f8f6f4), issued by one thread.
__device__ __forceinline__ void mma_f8_ss(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

}  // namespace

// The fused decode step's token and caches (FUSED only).
struct DecodeAppend {
  const uint4* k;           // the token's K and V rows [Hkv][hd] f16 and indexer key [d] f16
  const uint4* v;
  const uint4* idx;
  uint4* k_cache;           // caches (K/V in f16, or e4m3 codes with kv_scales)
  uint4* v_cache;
  uint4* idx_cache;
  PooledOut pooled;         // the pooled cache the TMA maps describe (f16, or e4m3 + scales)
  const float* gain;        // RMS-norm gain or null
  float* kv_scales;
  PoolRope rope;
  float eps;
  int kv_units, max_ctx, n_kv_heads, head_dim, fp8, gen;
};

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Warp 6 of the CTA that owns the last rows, in a decode step: after the dependency wait,
// appends the token at position n_old (K/V rows, FP8-quantised when the cache is, and the
// raw indexer key) and, when the token completes block b = (n_old + 1)/4 - 1, pools that
// block from its first three cached keys and the token's own key, writes the summary and
// makes it visible to the TMA loads (proxy fence, then an arrival on pool_bar). The
// summary is bit-identical to the one the pooling kernels compute.
template <int D, bool GEN>
__device__ __forceinline__ void decode_append_pool(const DecodeAppend& a, DevState* st, uint64_t* pool_bar,
                                                   float* s_row, int lane) {
  const PoolLane<D, GEN> c = pool_lane_consts<D, GEN>(lane, a.gain, a.rope.base, a.rope.dims, a.rope.interleaved);
  pdl_wait();
  const int n_old = ld_volatile(&st->n_ctx);
  const int n_pooled = ld_volatile(&st->n_pooled);
  if (n_old < 0 || n_old >= a.max_ctx || n_pooled != n_old / kBlock) return;  // the grid skips (reported there)
  if (!a.fp8) {
    for (int i = lane; i < a.kv_units; i += 32) {
      a.k_cache[size_t(n_old) * a.kv_units + i] = a.k[i];
      a.v_cache[size_t(n_old) * a.kv_units + i] = a.v[i];
    }
  } else {
    const __half* kh = reinterpret_cast<const __half*>(a.k);
    const __half* vh = reinterpret_cast<const __half*>(a.v);
    for (int r = 0; r < 2 * a.n_kv_heads; ++r) {
      const KvRow kr = kv_row(r, size_t(n_old), kh, vh, reinterpret_cast<unsigned char*>(a.k_cache),
                              reinterpret_cast<unsigned char*>(a.v_cache), a.kv_scales, a.n_kv_heads, a.head_dim);
      fp8_row_store(fp8_row_load(kr.src, a.head_dim, lane), kr.dst, kr.scale, a.head_dim, lane);
    }
  }
  constexpr int IDX_UNITS = D * 2 / 16;
  if (lane < IDX_UNITS) a.idx_cache[size_t(n_old) * IDX_UNITS + lane] = a.idx[lane];
  const int n = n_old + 1;
  if (n % kBlock) return;
  const int b = n / kBlock - 1;
  // raw keys of the block: three cached rows, then the token's own key (from the input)
  PoolRaw<D> raw;
  constexpr int P = D / 64, HALF = D / 2;
  const __half* ic = reinterpret_cast<const __half*>(a.idx_cache);
  const __half* key = reinterpret_cast<const __half*>(a.idx);
#pragma unroll
  for (int t = 0; t < kBlock; ++t) {
    const __half* row = t < kBlock - 1 ? ic + (size_t(b) * kBlock + t) * D : key;
    if constexpr (P == 2) {
      raw.x1[t] = *reinterpret_cast<const __half2*>(row + lane * 2);
      raw.x2[t] = *reinterpret_cast<const __half2*>(row + lane * 2 + HALF);
    } else {
      raw.x1[t] = __halves2half2(row[lane], __float2half_rn(0.0f));
      raw.x2[t] = __halves2half2(row[lane + HALF], __float2half_rn(0.0f));
    }
  }
  pool_finish<D, GEN>(b, lane, c, raw, a.pooled, a.eps, a.rope.pos, s_row);
  fence_proxy_async_global();  // the summary, written through the generic proxy, is read by TMA
  __syncwarp();
  if (lane == 0) mbar_arrive(pool_bar);
}

template <int D, int H, int T, bool HIST, bool FUSED, bool F8>
__global__ void __launch_bounds__(kThreads, 1)
index_scan_tc_kernel(const __grid_constant__ CUtensorMap map_tile, const __grid_constant__ CUtensorMap map_box,
                     DevState* st, const __half* __restrict__ q_idx, const float* __restrict__ w,
                     float* __restrict__ scores, uint32_t* __restrict__ hist, float rope_base, int max_blocks,
                     int rope_dims, int rope_interleaved, int rope_pos_stride, int score_stride, DecodeAppend app,
                     int q_n, const float* pooled_scales, int early) {
  static_assert(!FUSED || T == 1, "the fused append serves the single-query step");
  static_assert(!FUSED || HIST, "the decode step always fills the histogram");
  using S = ScanShape<D, H, T, F8>;
  constexpr int kAcc = S::ACC;
  constexpr int kStages = S::STAGES;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  unsigned char* sA = smem;
  unsigned char* sB = sA + size_t(kStages) * S::TILE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + S::B_BYTES);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + kAcc;
  uint64_t* pool_bar = tempty + kAcc;
  uint64_t* spec_bar = pool_bar + 1;  // the first tile loaded at the hinted range
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(spec_bar + 1);
  float* s_qmax = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(full) + 192);  // [4] (8-bit keys)
  int* s_nspec = reinterpret_cast<int*>(reinterpret_cast<unsigned char*>(full) + 208);     // early B operand
  static_assert((2 * kStages + 2 * kAcc + 2) * 8 + 4 <= 192, "barriers below the query-max slots");
  float* s_cos = reinterpret_cast<float*>(smem + size_t(kStages) * S::TILE_BYTES + S::B_BYTES + 256);
  float* s_sin = s_cos + T * (D / 2);                                 // [T][D/2] each
  double* s_theta = reinterpret_cast<double*>(s_sin + T * (D / 2));   // D/2 doubles
  __half* s_q = reinterpret_cast<__half*>(s_theta + D / 2);           // raw queries, T x H x D
  uint32_t* s_hist = reinterpret_cast<uint32_t*>(s_q + T * H * D);    // [T][kHistBins]
  float* s_row = reinterpret_cast<float*>(s_hist + T * kHistBins);    // [D] (pooling, generic RoPE)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_launch_dependents();
  if (threadIdx.x == 0) QSA_TL(st, kTlScan, kTlEntry);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < kAcc; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(pool_bar, 1);
    mbar_init(spec_bar, 1);
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_holder, S::TMEM_COLS);
    tmem_relinquish();
  }
  int spec_r0 = 0, spec_r1 = 0;  // warp 4 lane 0: this CTA's range at the hinted length
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&map_tile);
    tma_prefetch_desc(&map_box);
    // Start HBM -> L2 streaming of this CTA's rows while the previous kernels still run:
    // the context length read here, before the dependency wait, may be one token stale,
    // which only shifts the prefetched range slightly. Prefetches change nothing that
    // later loads observe; the real loads below use the current length.
    const int nb_hint = min(max(ld_volatile(&st->n_ctx) + (FUSED ? 1 : 0), 0) / kBlock, max_blocks);
    const int p0 = int((long long)blockIdx.x * nb_hint / gridDim.x);
    const int p1 = int((long long)(blockIdx.x + 1) * nb_hint / gridDim.x);
    spec_r0 = p0;
    spec_r1 = p1;
    for (int r = p0; r < p1; r += 128)
#pragma unroll
      for (int j = 0; j < S::HALVES; ++j) tma_prefetch_l2_2d(&map_tile, j * (128 / S::ESIZE), r);
  }
  // TMA loads of `rows` pooled rows from row0 into ring stage s, completing on bar
  auto issue_tile = [&](int s, int row0, int rows, uint64_t* bar) {
    unsigned char* dst = sA + size_t(s) * S::TILE_BYTES;
    if (rows == 128) {  // whole tile: one 128-row box per 128-byte span
      mbar_arrive_expect_tx(bar, uint32_t(S::TILE_BYTES));
#pragma unroll
      for (int j = 0; j < S::HALVES; ++j)
        tma_load_2d(dst + j * S::HALF_BYTES, &map_tile, j * (128 / S::ESIZE), row0, bar);
    } else {            // ragged tail: 16-row boxes, at most 15 rows past the range
      const int boxes = (rows + kBoxRows - 1) / kBoxRows;
      mbar_arrive_expect_tx(bar, uint32_t(boxes * kBoxRows * 128 * S::HALVES));
#pragma unroll
      for (int j = 0; j < S::HALVES; ++j)
        for (int b = 0; b < boxes; ++b)
          tma_load_2d(dst + j * S::HALF_BYTES + b * kBoxRows * 128, &map_box, j * (128 / S::ESIZE),
                      row0 + b * kBoxRows, bar);
    }
  };
  // RoPE frequencies do not depend on the previous kernel: compute them before waiting on it
  for (int i = threadIdx.x; i < rope_dims / 2; i += blockDim.x)
    s_theta[i] = pow((double)rope_base, -2.0 * (double)i / (double)rope_dims);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  // ---- warps 0-3: the B operand, the query rotated at the position of token n_pos - 1
  // (its last query) and split (f16 high and low parts, or e4m3 terms) ----
  const int tid = threadIdx.x;  // 0..127 in warps 0-3
  float pre = 1.0f;             // 8-bit keys: the query's power-of-2 prescale
  auto build_b = [&](int n_pos) {
    // raw queries: T*H*D f16 = T*H*D/8 16-byte vectors, all loads in flight at once
    constexpr int QV = T * H * D / 8;
    uint4 qraw[(QV + 127) / 128];
#pragma unroll
    for (int k = 0; k < (QV + 127) / 128; ++k)
      if (tid + k * 128 < QV) qraw[k] = reinterpret_cast<const uint4*>(q_idx)[tid + k * 128];
    if constexpr (F8) {  // largest |raw query element|: sets the power-of-2 prescale below
      float m = 0.0f;
#pragma unroll
      for (int k = 0; k < (QV + 127) / 128; ++k)
        if (tid + k * 128 < QV) {
          const __half2* hv = reinterpret_cast<const __half2*>(&qraw[k]);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __half22float2(hv[i]);
            m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
          }
        }
      m = warp_max(m);
      if (lane == 0) s_qmax[warp] = m;
    }
    // query u belongs to token n_pos - T + u: on the block-position scale it sits at
    // floor(stride * (n_u - 1) / 4), n_u = n_pos - T + u + 1 (token n_u - 1 when stride = 4)
    const int half_r = rope_dims / 2;
    for (int i = tid; i < T * half_r; i += 128) {
      const int u = i / half_r, f = i % half_r;
      const int n_u = n_pos - (T - 1 - u);
      const double qpos = n_u > 0 ? (double)(((long long)rope_pos_stride * (n_u - 1)) / kBlock) : 0.0;
      double sd, cd;
      sincos(qpos * s_theta[f], &sd, &cd);
      s_cos[u * (D / 2) + f] = (float)cd;
      s_sin[u * (D / 2) + f] = (float)sd;
    }
    if (tid == 0) QSA_TL(st, kTlScan2, 1);  // this thread's sin/cos done
#pragma unroll
    for (int k = 0; k < (QV + 127) / 128; ++k)
      if (tid + k * 128 < QV) reinterpret_cast<uint4*>(s_q)[tid + k * 128] = qraw[k];
    if (tid == 0) QSA_TL(st, kTlScan2, 0);  // this thread's query loads landed
    named_bar_sync(2, 128);
    // 8-bit keys: the rotated query times pre = 2^k, k set so that the largest raw element
    // lands in [64, 128); a rotated element is at most sqrt(2) times that, inside e4m3's
    // range (448). Each element becomes kF8Terms e4m3 terms, x_0 = pre * q~,
    // v_t = e4m3(x_t), x_{t+1} = (x_t - v_t) * 16 (both steps exact in f32), so that
    // pre * q~ = sum_t v_t 16^-t up to the last term's rounding (~2^-20 relative); term t
    // of head h is B row t*H + h and its dots are weighted by 16^-t in the epilogue.
    pre = 1.0f;
    if constexpr (F8) {
      const float m = fmaxf(fmaxf(s_qmax[0], s_qmax[1]), fmaxf(s_qmax[2], s_qmax[3]));
      int ex = 0;
      (void)frexpf(m, &ex);
      if (m > 0.0f) pre = ldexpf(1.0f, 7 - ex);
    }
    // rotated element e of head h of query u -> f16: high part in B row u*NQ + h, scaled
    // residual in row u*NQ + H + h; e4m3: terms in rows t*H + h
    auto put = [&](int u, int h, int e, float r) {
      if constexpr (F8) {
        float x = r * pre;
#pragma unroll
        for (int t = 0; t < kF8Terms; ++t) {
          const __nv_fp8_storage_t v = __nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
          sB[sw128_offset_b(t * H + h, e)] = v;
          x = (x - __half2float(__half(__nv_cvt_fp8_to_halfraw(v, __NV_E4M3)))) * 16.0f;
        }
      } else {
        const __half hi = __float2half_rn(r);
        const __half lo = __float2half_rn((r - __half2float(hi)) * kLoScale);
        *reinterpret_cast<__half*>(sB + sw128_offset(u * S::NQ + h, e, S::B_HALF_BYTES)) = hi;
        *reinterpret_cast<__half*>(sB + sw128_offset(u * S::NQ + H + h, e, S::B_HALF_BYTES)) = lo;
      }
    };
    if (rope_dims == D && !rope_interleaved) {  // NeoX pairs (i, i + D/2) over all dims
      for (int e = tid; e < T * H * (D / 2); e += 128) {
        const int uh = e / (D / 2), i = e % (D / 2);
        const int u = uh / H, h = uh % H;
        const __half* x = s_q + uh * D;
        const float c = s_cos[u * (D / 2) + i], sn = s_sin[u * (D / 2) + i];
        const float x1 = __half2float(x[i]);
        const float x2 = __half2float(x[i + D / 2]);
        put(u, h, i, x1 * c - x2 * sn);
        put(u, h, i + D / 2, x1 * sn + x2 * c);
      }
    } else {  // partial rotary or interleaved pairs: one element at a time
      for (int e = tid; e < T * H * D; e += 128) {
        const int uh = e / D, k = e % D;
        const int u = uh / H, h = uh % H;
        const __half* x = s_q + uh * D;
        const RopeSlot sl = rope_slot(k, rope_dims, rope_interleaved != 0);
        const float xk = __half2float(x[k]);
        float r = xk;
        if (sl.freq >= 0)
          r = xk * s_cos[u * (D / 2) + sl.freq] + sl.sign * __half2float(x[sl.partner]) * s_sin[u * (D / 2) + sl.freq];
        put(u, h, k, r);
      }
    }
    constexpr int USED = S::TERMS * H;
    constexpr int PAD = S::NQ - USED;  // zero rows after each query's term rows
    if constexpr (PAD > 0) {
      for (int e = tid; e < T * PAD * D; e += 128) {
        const int u = e / (PAD * D), rem = e % (PAD * D);
        if constexpr (F8) sB[sw128_offset_b(USED + rem / D, rem % D)] = 0;
        else
          *reinterpret_cast<__half*>(sB + sw128_offset(u * S::NQ + USED + rem / D, rem % D, S::B_HALF_BYTES)) =
              __float2half_rn(0.0f);
      }
    }
  };
  float wr[T][H];  // indexer head weights
  auto load_w = [&]() {
#pragma unroll
    for (int u = 0; u < T; ++u)
#pragma unroll
      for (int h = 0; h < H; ++h) wr[u][h] = w[u * H + h];
  };
  // Inputs complete at launch (early): build the B operand and load the weights before the
  // dependency wait, at the position the state holds now (the previous kernel on the stream
  // does not change it, except in a sequence like append-then-scan of the same layer, where
  // the position is checked after the wait and the operand rebuilt).
  int pos_built = -1;
  if (early && warp < 4) {
    if (tid == 0) *s_nspec = ld_volatile(&st->n_ctx) + (FUSED ? 1 : 0);
    named_bar_sync(2, 128);
    pos_built = q_n > 0 ? q_n : *s_nspec;
    build_b(pos_built);
    load_w();
  }
  if (warp < 4 && HIST)
    for (int i = tid; i < T * kHistBins; i += 128) s_hist[i] = 0u;


  if (FUSED && warp == 6) {
    // ---------------- warp 6: the decode step's append and new-block pooling ----------------
    if (blockIdx.x == gridDim.x - 1) {
      if (app.gen) decode_append_pool<D, true>(app, st, pool_bar, s_row, lane);
      else decode_append_pool<D, false>(app, st, pool_bar, s_row, lane);
    } else {
      pdl_wait();
    }
  }
  if (!(FUSED && warp == 6)) pdl_wait();
  if (threadIdx.x == 0) QSA_TL(st, kTlScan, kTlWait);
  // The first tile at the hinted range, issued now (the data is safe to read: the wait is
  // behind us) instead of after the state read; it is used only if the state confirms the
  // range. Not in the CTA whose rows a decode step's new block may join.
  bool spec_issued = false, spec_done = false;
  if (warp == 4 && lane == 0 && spec_r1 > spec_r0 && !(FUSED && blockIdx.x == gridDim.x - 1)) {
    issue_tile(0, spec_r0, min(128, spec_r1 - spec_r0), spec_bar);
    spec_issued = true;
  }
  const int n_old = ld_volatile(&st->n_ctx);
  const int n_pooled = ld_volatile(&st->n_pooled);
  // tokens the (last) query sees; the decode step's token is appended by this kernel
  const int n = FUSED ? n_old + 1 : n_old;
  bool state_ok = n_pooled == n_old / kBlock;
  if (FUSED) state_ok = state_ok && n_old >= 0 && n_old < app.max_ctx;
  if (!state_ok && blockIdx.x == 0 && threadIdx.x == 0)
    record_status(st, FUSED && (n_old >= app.max_ctx) ? QSA_ERR_CAPACITY : QSA_ERR_STATE);
  const int n_blocks = n / kBlock;
  const int r0 = int((long long)blockIdx.x * n_blocks / gridDim.x);
  const int r1 = int((long long)(blockIdx.x + 1) * n_blocks / gridDim.x);
  const int n_rows = state_ok ? r1 - r0 : 0;
  const int n_tiles = (n_rows + 127) / 128;
  // the tile that holds the block this step completes (last CTA of a fused step), or -1
  const int pool_tile = (FUSED && state_ok && n % kBlock == 0 && blockIdx.x == gridDim.x - 1)
                            ? (n_blocks - 1 - r0) / 128 : -1;

  if (n_tiles > 0 && warp < 6) {
    if (warp == 4) {
      // ---------------- TMA producer ----------------
      if (lane == 0) {
        int issued = 0;
        bool ok = true;
        for (int t = 0; t < n_tiles && ok; ++t) {
          const int s = t % kStages;
          if (t >= kStages && !mbar_wait(&empty[s], ((t / kStages) - 1) & 1)) {
            ok = false;
            break;
          }
          if (FUSED && t == pool_tile && !mbar_wait(pool_bar, 0)) {  // the new summary is in memory
            ok = false;
            break;
          }
          if (t == 0 && spec_issued) {
            spec_done = true;
            if (!mbar_wait(spec_bar, 0)) {  // the early tile has landed, whatever its rows
              ok = false;
              break;
            }
            if (spec_r0 == r0 && spec_r1 == r0 + n_rows) {  // the hinted range was right
              mbar_arrive(&full[0]);
              QSA_TL(st, kTlScan2, 3);
              ++issued;
              continue;
            }
          }
          issue_tile(s, r0 + t * 128, min(128, n_rows - t * 128), &full[s]);
          if (t == 0) QSA_TL(st, kTlScan2, 3);  // first tile's loads issued
          ++issued;
        }
        if (!ok) record_status(st, QSA_ERR_TIMEOUT);
        // every fill this thread started must land before the CTA's shared memory is released
        for (int t = max(0, issued - kStages); t < issued; ++t) mbar_wait(&full[t % kStages], (t / kStages) & 1);
        if (spec_issued && !spec_done) mbar_wait(spec_bar, 0);
        spec_done = true;
      }
    } else if (warp == 5) {
      // ---------------- MMA issuer ----------------
      named_bar_sync(1, 160);  // B operand written by warps 0-3
      if (lane == 0) {
        bool ok = true;
        int last = -1;
        for (int t = 0; t < n_tiles; ++t) {
          const int s = t % kStages, a = t % kAcc;
          if (!mbar_wait(&full[s], (t / kStages) & 1)) { ok = false; break; }
          if (t == 0) QSA_TL(st, kTlScan, kTlA);  // first tile landed
          if (t >= kAcc && !mbar_wait(&tempty[a], ((t / kAcc) - 1) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + uint32_t(a * S::N);
          const uint32_t a0 = smem_u32(sA + size_t(s) * S::TILE_BYTES);
          const uint32_t b0 = smem_u32(sB);
#pragma unroll
          for (int kk = 0; kk < S::K_STEPS; ++kk) {
            const int j = kk >> 2, kin = kk & 3;  // 128-byte span, 32-byte K step inside it
            const uint64_t adesc = smem_desc_sw128(a0 + j * S::HALF_BYTES + kin * 32);
            const uint64_t bdesc = smem_desc_sw128(b0 + j * S::B_HALF_BYTES + kin * 32);
            if constexpr (F8) mma_f8_ss(d_tmem, adesc, bdesc, S::IDESC, kk > 0 ? 1u : 0u);
            else mma_f16_ss(d_tmem, adesc, bdesc, S::IDESC, kk > 0 ? 1u : 0u);
          }
          tc_commit(&empty[s]);
          tc_commit(&tfull[a]);
          last = t;
        }
        if (last >= 0) QSA_TL(st, kTlScan2, 4);  // last tile's MMAs issued
        if (!ok) record_status(st, QSA_ERR_TIMEOUT);
        // the tensor core must be done with TMEM before it is freed
        if (last >= 0) mbar_wait(&tfull[last % kAcc], (last / kAcc) & 1);
      }
      __syncwarp();
    } else {
      // ---------------- warps 0-3: rotated, split query -> B operand; then epilogue ----------------
      // the query's position: q_n > 0 when it belongs to token q_n - 1 of a longer sequence
      // whose blocks this layer holds a contiguous part of (a context-parallel shard)
      const int pos = q_n > 0 ? q_n : n;  // uniform
      if (pos != pos_built) {
        if (pos_built >= 0) named_bar_sync(2, 128);  // every thread is done with the first build
        build_b(pos);
        load_w();
      }
      fence_proxy_async_smem();
      named_bar_sync(1, 160);
      if (tid == 0) QSA_TL(st, kTlScan2, 2);  // B operand built

      const float sqrt_d = sqrtf((float)D);
      const float unscale = 1.0f / pre;  // a power of 2: exact
      bool ok = true;
      for (int t = 0; t < n_tiles; ++t) {
        const int a = t % kAcc;
        const int row = r0 + t * 128 + tid;
        // 8-bit keys: the row's scale (the block this step pools: once warp 6 has written it)
        float row_scale = 1.0f;
        if constexpr (F8)
          if (row < r1 && t != pool_tile) row_scale = pooled_scales[row];
        if (!mbar_wait(&tfull[a], (t / kAcc) & 1)) { ok = false; break; }
        if constexpr (F8)
          if (row < r1 && t == pool_tile && mbar_wait(pool_bar, 0)) row_scale = pooled_scales[row];
        tc_fence_after();
        const uint32_t taddr = tmem_base + (uint32_t(32 * warp) << 16) + uint32_t(a * S::N);
        uint32_t r[T][S::NQ];  // query u's columns [u*NQ, (u+1)*NQ) of this row
#pragma unroll
        for (int u = 0; u < T; ++u) {
#pragma unroll
          for (int c = 0; c < S::NQ / 32; ++c)
            tmem_ld_32x32b_x32(taddr + uint32_t(u * S::NQ + 32 * c), reinterpret_cast<uint32_t(&)[32]>(r[u][32 * c]));
          if constexpr (S::NQ % 32 != 0)
            tmem_ld_32x32b_x16(taddr + uint32_t(u * S::NQ + S::NQ / 32 * 32),
                               reinterpret_cast<uint32_t(&)[16]>(r[u][S::NQ / 32 * 32]));
        }
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&tempty[a]);
        if (row < r1) {
#pragma unroll
          for (int u = 0; u < T; ++u) {
            float s = 0.0f;
#pragma unroll
            for (int h = 0; h < H; ++h) {
              float dot;
              if constexpr (F8) {  // sum_t acc_t 16^-t, smallest term first
                dot = __uint_as_float(r[u][(kF8Terms - 1) * H + h]);
#pragma unroll
                for (int tt = kF8Terms - 2; tt >= 0; --tt) dot = fmaf(dot, 1.0f / 16.0f, __uint_as_float(r[u][tt * H + h]));
              } else {
                dot = __uint_as_float(r[u][h]) + __uint_as_float(r[u][H + h]) * (1.0f / kLoScale);
              }
              s += wr[u][h] * fmaxf(dot, 0.0f);
            }
            // 8-bit keys: the dots were of pre * q~ with the codes; scale and prescale are
            // positive, so they come out of the max(0, .) unchanged
            const float score = F8 ? s * (row_scale * unscale) / sqrt_d : s / sqrt_d;
            scores[size_t(u) * score_stride + row] = score;
            // query u counts only the blocks its own n_u = n - (T-1-u) tokens complete
            if constexpr (HIST)
              if (row < (n - (T - 1 - u)) / kBlock)
                atomicAdd(&s_hist[u * kHistBins + (sel::score_key(score) >> (32 - kHistBits))], 1u);
          }
        }
      }
      if (!ok && tid == 0) record_status(st, QSA_ERR_TIMEOUT);
      if (tid == 0) QSA_TL(st, kTlScan, kTlB);  // this thread's rows scored
      if constexpr (HIST) {  // this CTA's counts into the layer's histogram
        named_bar_sync(2, 128);
        // thread t: kPer consecutive bins, read 4 at a time, one reduction per non-zero
        // bin; query u's bins sit at hist + u * kHistBins
        constexpr int kPer = T * kHistBins / 128;
        static_assert(kPer % 4 == 0, "whole 16-byte vectors");
#pragma unroll 1
        for (int v = 0; v < kPer / 4; ++v) {
          const uint4 c4 = reinterpret_cast<const uint4*>(s_hist + tid * kPer)[v];
          uint32_t* dst = hist + tid * kPer + 4 * v;
          if (c4.x) atomicAdd(dst, c4.x);
          if (c4.y) atomicAdd(dst + 1, c4.y);
          if (c4.z) atomicAdd(dst + 2, c4.z);
          if (c4.w) atomicAdd(dst + 3, c4.w);
        }
        if (tid == 0) QSA_TL(st, kTlScan3, 0);  // histogram flushed (this thread's part)
      }
    }
  }
  if (spec_issued && !spec_done) mbar_wait(spec_bar, 0);  // no tiles here: the early tile lands first
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) QSA_TL(st, kTlScan3, 1);  // every warp done
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem_base, S::TMEM_COLS);
  }
  if (threadIdx.x == 0) QSA_TL(st, kTlScan, kTlExit);
}

// ---------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------
template <int D, int H, int T, bool HIST, bool FUSED, bool F8 = false>
static cudaError_t set_scan_attr() {
  cudaError_t e = cudaFuncSetAttribute(index_scan_tc_kernel<D, H, T, HIST, FUSED, F8>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)ScanShape<D, H, T, F8>::SMEM);
  if (e == cudaSuccess)  // the whole unified L1/shared array as shared memory (see qsa_device.cuh)
    e = cudaFuncSetAttribute(index_scan_tc_kernel<D, H, T, HIST, FUSED, F8>,
                             cudaFuncAttributePreferredSharedMemoryCarveout, kCarveoutMaxShared);
  return e;
}

template <int D, int H>
static cudaError_t set_scan_attr_t() {
  cudaError_t e;
  if ((e = set_scan_attr<D, H, 1, false, false>()) != cudaSuccess ||
      (e = set_scan_attr<D, H, 1, true, false>()) != cudaSuccess ||
      (e = set_scan_attr<D, H, 1, true, true>()) != cudaSuccess ||
      (e = set_scan_attr<D, H, 2, false, false>()) != cudaSuccess ||
      (e = set_scan_attr<D, H, 3, false, false>()) != cudaSuccess ||
      (e = set_scan_attr<D, H, 4, false, false>()) != cudaSuccess ||
      (e = set_scan_attr<D, H, 2, true, false>()) != cudaSuccess ||
      (e = set_scan_attr<D, H, 3, true, false>()) != cudaSuccess ||
      (e = set_scan_attr<D, H, 4, true, false>()) != cudaSuccess)
    return e;
  if constexpr (D == 128) {  // 8-bit pooled keys: single query
    if ((e = set_scan_attr<D, H, 1, false, false, true>()) != cudaSuccess ||
        (e = set_scan_attr<D, H, 1, true, false, true>()) != cudaSuccess ||
        (e = set_scan_attr<D, H, 1, true, true, true>()) != cudaSuccess)
      return e;
  }
  return cudaSuccess;
}

cudaError_t init_scan_attributes() {
  static_assert(kMaxQueries == 4, "one scan instantiation per query count");
  cudaError_t e = cudaSuccess;
#define QSA_SCAN_ATTR(DD)                                                                                 \
  if ((e = set_scan_attr_t<DD, 1>()) != cudaSuccess || (e = set_scan_attr_t<DD, 2>()) != cudaSuccess ||   \
      (e = set_scan_attr_t<DD, 4>()) != cudaSuccess || (e = set_scan_attr_t<DD, 8>()) != cudaSuccess ||   \
      (e = set_scan_attr_t<DD, 16>()) != cudaSuccess)                                                     \
    return e;
  QSA_SCAN_ATTR(64)
  QSA_SCAN_ATTR(128)
#undef QSA_SCAN_ATTR
  return e;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// TMA descriptor of a layer's pooled cache: rows = max_ctx/4 blocks of d_idx f16 (or e4m3
// codes with QSA_POOLED_FP8), box_rows x 128-byte boxes written with the 128-byte swizzle.
cudaError_t encode_pooled_map(const qsa_config& c, void* pooled, int box_rows, CUtensorMap* out) {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (e != cudaSuccess) return e;
    if (q != cudaDriverEntryPointSuccess || !p) return cudaErrorNotSupported;
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  const cuuint64_t dims[2] = {cuuint64_t(c.d_idx), cuuint64_t(c.max_ctx / kBlock)};
  const bool fp8 = c.pooled_format == QSA_POOLED_FP8;
  const cuuint64_t strides[1] = {cuuint64_t(c.d_idx) * (fp8 ? 1 : 2)};
  const cuuint32_t box[2] = {fp8 ? 128u : 64u, cuuint32_t(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(out, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, pooled, dims,
                        strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int D, int H, int T, bool HIST, bool FUSED, bool F8 = false>
static cudaError_t launch_scan_tc(const LayerView& L, const void* q_idx, const float* w, float* scores,
                                  cudaStream_t s, int score_stride, uint32_t* hist, const DecodeAppend& app,
                                  int q_n = 0) {
  return launch_pdl(index_scan_tc_kernel<D, H, T, HIST, FUSED, F8>, dim3(L.n_sms), dim3(kThreads),
                    ScanShape<D, H, T, F8>::SMEM, s, 1, L.pooled_tile_map, L.pooled_box_map, L.state,
                    (const __half*)q_idx, w, scores, hist, L.cfg.rope_base, L.cfg.max_ctx / kBlock, L.cfg.rope_dims,
                    L.cfg.rope_interleaved, L.cfg.rope_pos_stride, score_stride, app, q_n,
                    (const float*)L.pooled_scales, L.cfg.early_inputs);
}

// mode 0: plain scan of T queries; 1: single query with the histogram; 2: decode step
template <int D, int H>
static cudaError_t launch_scan_tc_t(const LayerView& L, const void* q_idx, const float* w, float* scores,
                                    cudaStream_t s, int n_queries, int score_stride, uint32_t* hist, int mode,
                                    const DecodeAppend& app, int q_n) {
  if (L.cfg.pooled_format == QSA_POOLED_FP8) {  // single query (checked by the callers)
    if constexpr (D == 128) {
      if (n_queries != 1) return cudaErrorInvalidValue;
      if (mode == 2) return launch_scan_tc<D, H, 1, true, true, true>(L, q_idx, w, scores, s, score_stride, hist, app);
      if (mode == 1)
        return launch_scan_tc<D, H, 1, true, false, true>(L, q_idx, w, scores, s, score_stride, hist, app, q_n);
      return launch_scan_tc<D, H, 1, false, false, true>(L, q_idx, w, scores, s, score_stride, hist, app, q_n);
    }
    return cudaErrorInvalidValue;
  }
  if (mode == 2) return launch_scan_tc<D, H, 1, true, true>(L, q_idx, w, scores, s, score_stride, hist, app);
  if (mode == 1) {  // with the score-key histograms (one per query)
    switch (n_queries) {
      case 1: return launch_scan_tc<D, H, 1, true, false>(L, q_idx, w, scores, s, score_stride, hist, app, q_n);
      case 2: return launch_scan_tc<D, H, 2, true, false>(L, q_idx, w, scores, s, score_stride, hist, app);
      case 3: return launch_scan_tc<D, H, 3, true, false>(L, q_idx, w, scores, s, score_stride, hist, app);
      case 4: return launch_scan_tc<D, H, 4, true, false>(L, q_idx, w, scores, s, score_stride, hist, app);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (n_queries) {
    case 1: return launch_scan_tc<D, H, 1, false, false>(L, q_idx, w, scores, s, score_stride, hist, app, q_n);
    case 2: return launch_scan_tc<D, H, 2, false, false>(L, q_idx, w, scores, s, score_stride, hist, app);
    case 3: return launch_scan_tc<D, H, 3, false, false>(L, q_idx, w, scores, s, score_stride, hist, app);
    case 4: return launch_scan_tc<D, H, 4, false, false>(L, q_idx, w, scores, s, score_stride, hist, app);
    default: return cudaErrorInvalidValue;
  }
}

template <int D>
static cudaError_t launch_scan_tc_d(const LayerView& L, const void* q_idx, const float* w, float* scores,
                                    cudaStream_t s, int n_queries, int score_stride, uint32_t* hist, int mode,
                                    const DecodeAppend& app, int q_n) {
  switch (L.cfg.n_idx_heads) {
    case 1: return launch_scan_tc_t<D, 1>(L, q_idx, w, scores, s, n_queries, score_stride, hist, mode, app, q_n);
    case 2: return launch_scan_tc_t<D, 2>(L, q_idx, w, scores, s, n_queries, score_stride, hist, mode, app, q_n);
    case 4: return launch_scan_tc_t<D, 4>(L, q_idx, w, scores, s, n_queries, score_stride, hist, mode, app, q_n);
    case 8: return launch_scan_tc_t<D, 8>(L, q_idx, w, scores, s, n_queries, score_stride, hist, mode, app, q_n);
    case 16: return launch_scan_tc_t<D, 16>(L, q_idx, w, scores, s, n_queries, score_stride, hist, mode, app, q_n);
    default: return cudaErrorInvalidValue;
  }
}

static cudaError_t launch_scan_mode(const LayerView& L, const void* q_idx, const float* w, float* scores,
                                    cudaStream_t s, int n_queries, int score_stride, uint32_t* hist, int mode,
                                    const DecodeAppend& app, int q_n = 0) {
  return L.cfg.d_idx == 128
             ? launch_scan_tc_d<128>(L, q_idx, w, scores, s, n_queries, score_stride, hist, mode, app, q_n)
             : launch_scan_tc_d<64>(L, q_idx, w, scores, s, n_queries, score_stride, hist, mode, app, q_n);
}

cudaError_t launch_index_scan(const LayerView& L, const void* q_idx, const float* w, float* scores,
                              cudaStream_t s, int n_queries, int score_stride, uint32_t* hist, int q_n) {
  if (L.cfg.scan_kind == QSA_SCAN_CUDA_CORES && n_queries == 1)
    return launch_index_scan_cc(L, q_idx, w, scores, hist, s, q_n);
  const int mode = hist ? 1 : 0;
  return launch_scan_mode(L, q_idx, w, scores, s, n_queries, score_stride, hist, mode, DecodeAppend{},
                          n_queries == 1 ? q_n : 0);
}

cudaError_t launch_decode_scan(const LayerView& L, const void* k, const void* v, const void* idx, const void* q_idx,
                               const float* w, float* scores, uint32_t* hist, cudaStream_t s) {
  DecodeAppend app{};
  app.k = static_cast<const uint4*>(k);
  app.v = static_cast<const uint4*>(v);
  app.idx = static_cast<const uint4*>(idx);
  app.k_cache = static_cast<uint4*>(L.k_cache);
  app.v_cache = static_cast<uint4*>(L.v_cache);
  app.idx_cache = static_cast<uint4*>(L.idx_cache);
  app.pooled = pooled_out(L);
  app.gain = L.rms_gain;
  app.kv_scales = L.kv_scales;
  app.rope = PoolRope{L.cfg.rope_base, L.cfg.rope_dims, L.cfg.rope_interleaved,
                      RopePos{L.cfg.rope_pos_stride, L.cfg.rope_pos_offset}};
  app.eps = L.cfg.rms_eps;
  app.kv_units = L.cfg.n_kv_heads * L.cfg.head_dim * 2 / 16;
  app.max_ctx = L.cfg.max_ctx;
  app.n_kv_heads = L.cfg.n_kv_heads;
  app.head_dim = L.cfg.head_dim;
  app.fp8 = L.cfg.kv_format == QSA_KV_FP8;
  app.gen = L.cfg.rope_dims != L.cfg.d_idx || L.cfg.rope_interleaved != 0;
  return launch_scan_mode(L, q_idx, w, scores, s, 1, 0, hist, 2, app);
}

}  // namespace qsa
