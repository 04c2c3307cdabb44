// Indexer scan on the CUDA cores (layer option scan_kind = QSA_SCAN_CUDA_CORES): the same
// scores as the tensor-core scan in qsa_scan_tc.cu, computed the way a GEMV-shaped
// memory-bound pass is usually written, kept as the measured alternative to it.
//
// Web page "Part 10" (第10回 EVO-X2 ... 長コンテキストのTGを高速化した話), section
// "QSA indexer": the current indexer query is scored against every completed block's
// pooled summary. This library's score (the pages give no formula):
//    score_b = sum_h w_h * max(0, q~_h . p_b) / sqrt(d),   q~_h = RoPE(q_h, n-1)
//
// Each CTA (one per SM) owns a contiguous range of pooled rows and streams it through a
// ring of shared-memory chunks with 1-D bulk copies (cp.async.bulk, completion on an
// mbarrier), the L2 prefetch issued before the dependency wait as in the tensor-core
// scan. A row of d f16 values is read by d/8 lanes, 16 bytes each; each lane keeps its
// slice of the rotated f32 query of every head in registers and accumulates its partial
// dots with packed f32 FMAs (fma.rn.f32x2), then a transposed shuffle reduction gives
// each lane the full dot of one head (or several), and a second one the weighted-ReLU
// sum. The query keeps full f32 precision (no f16 split).
#include <cuda_fp16.h>

#include "qsa_device.cuh"
#include "qsa_select.cuh"
#include "qsa_sm100.cuh"

namespace qsa {

namespace {

using namespace sm100;

constexpr int kCcThreads = 256;   // 8 warps
constexpr int kCcChunkRows = 64;  // rows per shared-memory chunk
constexpr int kCcStages = 8;      // chunks in the ring

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  unsigned long long ra, rb, rc, rd;
  ra = *reinterpret_cast<unsigned long long*>(&a);
  rb = *reinterpret_cast<unsigned long long*>(&b);
  rc = *reinterpret_cast<unsigned long long*>(&c);
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(rd) : "l"(ra), "l"(rb), "l"(rc));
  return *reinterpret_cast<float2*>(&rd);
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Sum of V per-lane values over groups of LPR consecutive lanes, transposed: afterwards
// lane l holds in v[0 .. max(V/LPR,1)) the group sums of the heads listed by head_of().
template <int V, int LPR>
__device__ __forceinline__ void group_transpose_reduce(float (&v)[V], int lane) {
#pragma unroll
  for (int half = V / 2, off = LPR / 2; half >= 1 && off >= 1; half >>= 1, off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? v[i] : v[i + half];
      const float keep = upper ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  if constexpr (V < LPR) {  // the remaining offsets add lanes holding the same head
#pragma unroll
    for (int off = LPR / (2 * V); off >= 1; off >>= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
  }
}

// Head of value i held by lane `lane` after group_transpose_reduce<V, LPR>.
template <int V, int LPR>
__device__ __forceinline__ int reduced_head(int lane, int i) {
  int h = i;
  int half = V / 2;
#pragma unroll
  for (int off = LPR / 2; off >= 1 && half >= 1; off >>= 1, half >>= 1) h += (lane & off) ? half : 0;
  return h;
}

}  // namespace

template <int D, int H, bool HIST>
__global__ void __launch_bounds__(kCcThreads, 1)
index_scan_cc_kernel(DevState* st, const __half* __restrict__ pooled, const __half* __restrict__ q_idx,
                     const float* __restrict__ w, float* __restrict__ scores, uint32_t* __restrict__ hist,
                     float rope_base, int max_blocks, int rope_dims, int rope_interleaved, int rope_pos_stride,
                     int q_n) {
  constexpr int LPR = D / 8;            // lanes per row (16 bytes each)
  constexpr int RPW = 32 / LPR;         // rows per warp per pass
  constexpr int NV = H < LPR ? 1 : H / LPR;  // reduced values per lane
  constexpr int kWarps = kCcThreads / 32;
  constexpr int CHUNK_BYTES = kCcChunkRows * D * 2;
  constexpr int kHB = 1 << kHistBits;
  extern __shared__ __align__(128) unsigned char smem[];
  __half* ring = reinterpret_cast<__half*>(smem);                                  // [stages][rows][D]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kCcStages * CHUNK_BYTES);    // [stages]
  float* s_q = reinterpret_cast<float*>(full + kCcStages);                         // [H][D] rotated query
  double* s_theta = reinterpret_cast<double*>(s_q + H * D);                         // [D/2]
  float* s_cs = reinterpret_cast<float*>(s_theta + D / 2);                          // [D/2] cos, [D/2] sin
  uint32_t* s_hist = reinterpret_cast<uint32_t*>(s_cs + D);                         // [kHB]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_launch_dependents();
  if (tid == 0) {
    for (int s = 0; s < kCcStages; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
    // HBM -> L2 streaming of this CTA's rows before the dependency wait (a hint only)
    const int nb_hint = min(max(ld_volatile(&st->n_ctx), 0) / kBlock, max_blocks);
    const int p0 = int((long long)blockIdx.x * nb_hint / gridDim.x);
    const int p1 = int((long long)(blockIdx.x + 1) * nb_hint / gridDim.x);
    for (int r = p0; r < p1; r += kCcChunkRows)
      bulk_prefetch_l2(pooled + size_t(r) * D, uint32_t(min(kCcChunkRows, p1 - r)) * D * 2);
  }
  for (int i = tid; i < rope_dims / 2; i += kCcThreads)
    s_theta[i] = pow((double)rope_base, -2.0 * (double)i / (double)rope_dims);
  if constexpr (HIST)
    for (int i = tid; i < kHB; i += kCcThreads) s_hist[i] = 0u;
  __syncthreads();

  pdl_wait();
  const int n = ld_volatile(&st->n_ctx);
  const int n_blocks = n / kBlock;
  const bool stale = ld_volatile(&st->n_pooled) != n_blocks;
  if (stale && blockIdx.x == 0 && tid == 0) record_status(st, QSA_ERR_STATE);
  const int r0 = int((long long)blockIdx.x * n_blocks / gridDim.x);
  const int r1 = int((long long)(blockIdx.x + 1) * n_blocks / gridDim.x);
  const int n_rows = stale ? 0 : r1 - r0;
  const int n_chunks = (n_rows + kCcChunkRows - 1) / kCcChunkRows;
  auto issue = [&](int c) {
    const int rows = min(kCcChunkRows, n_rows - c * kCcChunkRows);
    uint64_t* bar = &full[c % kCcStages];
    mbar_arrive_expect_tx(bar, uint32_t(rows) * D * 2);
    bulk_load(ring + size_t(c % kCcStages) * kCcChunkRows * D, pooled + size_t(r0 + c * kCcChunkRows) * D,
              uint32_t(rows) * D * 2, bar);
  };
  if (tid == 0)
    for (int c = 0; c < min(n_chunks, kCcStages); ++c) issue(c);

  // the rotated query (position of token n-1 on the block-position scale), f32
  const int half_r = rope_dims / 2;
  const int nq = q_n > 0 ? q_n : n;  // the query's token count (a shard's query sits in a longer sequence)
  const double qpos = nq > 0 ? (double)(((long long)rope_pos_stride * (nq - 1)) / kBlock) : 0.0;
  for (int f = tid; f < half_r; f += kCcThreads) {
    double sd, cd;
    sincos(qpos * s_theta[f], &sd, &cd);
    s_cs[f] = (float)cd;
    s_cs[D / 2 + f] = (float)sd;
  }
  __syncthreads();
  for (int e = tid; e < H * D; e += kCcThreads) {
    const int h = e / D, k = e % D;
    const __half* x = q_idx + size_t(h) * D;
    const RopeSlot sl = rope_slot(k, rope_dims, rope_interleaved != 0);
    const float xk = __half2float(x[k]);
    float r = xk;
    if (sl.freq >= 0) r = xk * s_cs[sl.freq] + sl.sign * __half2float(x[sl.partner]) * s_cs[D / 2 + sl.freq];
    s_q[h * D + k] = r;
  }
  __syncthreads();
  // this lane's 8 query elements of every head, as f32 pairs
  const int sub = lane % LPR;
  float2 qv[H][4];
#pragma unroll
  for (int h = 0; h < H; ++h)
#pragma unroll
    for (int k = 0; k < 4; ++k) qv[h][k] = *reinterpret_cast<const float2*>(s_q + h * D + sub * 8 + 2 * k);
  float wv[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) wv[i] = w[reduced_head<H, LPR>(lane, i)];
  const float inv_sqrt_d = 1.0f / sqrtf((float)D);

  bool ok = true;
  for (int c = 0; c < n_chunks; ++c) {
    const int slot = c % kCcStages;
    if (!mbar_wait(&full[slot], (c / kCcStages) & 1)) ok = false;
    const int rows = ok ? min(kCcChunkRows, n_rows - c * kCcChunkRows) : 0;
    const __half* chunk = ring + size_t(slot) * kCcChunkRows * D;
    for (int g = warp; g * RPW < rows; g += kWarps) {
      const int lr = g * RPW + lane / LPR;  // row within the chunk (same for the LPR lanes)
      uint4 raw = make_uint4(0u, 0u, 0u, 0u);
      if (lr < rows) raw = *reinterpret_cast<const uint4*>(chunk + size_t(lr) * D + sub * 8);
      const __half2* hp = reinterpret_cast<const __half2*>(&raw);
      float2 p[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) p[k] = __half22float2(hp[k]);
      float acc[H];
#pragma unroll
      for (int h = 0; h < H; ++h) {
        float2 a = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int k = 0; k < 4; ++k) a = ffma2(qv[h][k], p[k], a);
        acc[h] = a.x + a.y;
      }
      group_transpose_reduce<H, LPR>(acc, lane);
      float sv = 0.0f;
#pragma unroll
      for (int i = 0; i < NV; ++i) sv += wv[i] * fmaxf(acc[i], 0.0f);
      // sum over the lanes of the group that hold different heads: offsets LPR/2 down to
      // the smallest that separates heads (lanes below it hold copies of the same head)
      constexpr int kLowOff = H < LPR ? LPR / H : 1;
#pragma unroll
      for (int off = LPR / 2; off >= kLowOff; off >>= 1) sv += __shfl_xor_sync(0xffffffffu, sv, off);
      if (sub == 0 && lr < rows) {
        const float score = sv * inv_sqrt_d;
        scores[r0 + c * kCcChunkRows + lr] = score;
        if constexpr (HIST) atomicAdd(&s_hist[sel::score_key(score) >> (32 - kHistBits)], 1u);
      }
    }
    __syncthreads();  // every warp is done with this slot
    if (tid == 0 && ok && c + kCcStages < n_chunks) issue(c + kCcStages);
  }
  if (!ok && tid == 0) record_status(st, QSA_ERR_TIMEOUT);
  if (tid == 0) {
    // every copy this CTA started has landed before its shared memory is released
    for (int c = max(0, n_chunks - kCcStages); c < n_chunks; ++c) mbar_wait(&full[c % kCcStages], (c / kCcStages) & 1);
  }
  if constexpr (HIST) {
    __syncthreads();
    for (int i = tid; i < kHB; i += kCcThreads) {
      const uint32_t v = s_hist[i];
      if (v) atomicAdd(hist + i, v);
    }
  }
}

namespace {
template <int D, int H>
constexpr size_t cc_smem() {
  return size_t(kCcStages) * kCcChunkRows * D * 2 + kCcStages * 8 + H * D * 4 + D / 2 * 8 + D * 4 +
         (1 << kHistBits) * 4;
}

template <int D, int H>
cudaError_t set_cc_attr() {
  cudaError_t e = cudaFuncSetAttribute(index_scan_cc_kernel<D, H, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)cc_smem<D, H>());
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(index_scan_cc_kernel<D, H, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)cc_smem<D, H>());
  return e;
}

template <int D, int H>
cudaError_t launch_cc(const LayerView& L, const void* q_idx, const float* w, float* scores, uint32_t* hist,
                      cudaStream_t s, int q_n) {
  const auto args = [&](auto kernel) {
    return launch_pdl(kernel, dim3(L.n_sms), dim3(kCcThreads), cc_smem<D, H>(), s, 1, L.state,
                      (const __half*)L.pooled_cache, (const __half*)q_idx, w, scores, hist, L.cfg.rope_base,
                      L.cfg.max_ctx / kBlock, L.cfg.rope_dims, L.cfg.rope_interleaved, L.cfg.rope_pos_stride, q_n);
  };
  return hist ? args(index_scan_cc_kernel<D, H, true>) : args(index_scan_cc_kernel<D, H, false>);
}

template <int D>
cudaError_t launch_cc_d(const LayerView& L, const void* q_idx, const float* w, float* scores, uint32_t* hist,
                        cudaStream_t s, int q_n) {
  switch (L.cfg.n_idx_heads) {
    case 1: return launch_cc<D, 1>(L, q_idx, w, scores, hist, s, q_n);
    case 2: return launch_cc<D, 2>(L, q_idx, w, scores, hist, s, q_n);
    case 4: return launch_cc<D, 4>(L, q_idx, w, scores, hist, s, q_n);
    case 8: return launch_cc<D, 8>(L, q_idx, w, scores, hist, s, q_n);
    case 16: return launch_cc<D, 16>(L, q_idx, w, scores, hist, s, q_n);
    default: return cudaErrorInvalidValue;
  }
}
}  // namespace

cudaError_t init_scan_cc_attributes() {
  cudaError_t e;
  if ((e = set_cc_attr<64, 1>()) != cudaSuccess || (e = set_cc_attr<64, 2>()) != cudaSuccess ||
      (e = set_cc_attr<64, 4>()) != cudaSuccess || (e = set_cc_attr<64, 8>()) != cudaSuccess ||
      (e = set_cc_attr<64, 16>()) != cudaSuccess || (e = set_cc_attr<128, 1>()) != cudaSuccess ||
      (e = set_cc_attr<128, 2>()) != cudaSuccess || (e = set_cc_attr<128, 4>()) != cudaSuccess ||
      (e = set_cc_attr<128, 8>()) != cudaSuccess || (e = set_cc_attr<128, 16>()) != cudaSuccess)
    return e;
  return cudaSuccess;
}

cudaError_t launch_index_scan_cc(const LayerView& L, const void* q_idx, const float* w, float* scores,
                                 uint32_t* hist, cudaStream_t s, int q_n) {
  return L.cfg.d_idx == 128 ? launch_cc_d<128>(L, q_idx, w, scores, hist, s, q_n)
                            : launch_cc_d<64>(L, q_idx, w, scores, hist, s, q_n);
}

}  // namespace qsa
