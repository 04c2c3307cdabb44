// Indexer scan and block-domain top-k.
//
// Web page "Part 10" (第10回 EVO-X2 ... 長コンテキストのTGを高速化した話):
//  - section "QSA indexer": the current query is scored against every completed
//    block's pooled summary and the high-scoring blocks are chosen by top-k;
//  - section "block-domain top-k（COMMON-006）実装は見送り": select in the block domain,
//    then expand only the chosen blocks into cells (no expansion of every cell).
// Score (the pages give no formula; this library's definition):
//    score_b = sum_h w_h * max(0, RoPE(q_h, n-1) . p_b) / sqrt(d_idx)
// Top-k: the min(K, B) largest scores, ties to the lower block index, output ascending.
#include <cooperative_groups.h>
#include <cuda_fp16.h>

#include "qsa_device.cuh"

namespace cg = cooperative_groups;

namespace qsa {

// ---------------------------------------------------------------------------------
// Indexer scan on the CUDA cores. Each warp scores one block at a time (U blocks per
// iteration for memory-level parallelism): lane l holds dims [l*VPL, (l+1)*VPL) of the
// rotated query of every head, reads the same dims of the block's f16 summary (one
// coalesced 2*D-byte row per warp), and a transposing reduction gives each lane one
// head's dot product. Accumulation is f32.
// ---------------------------------------------------------------------------------
template <int D, int H>
__global__ void __launch_bounds__(256) index_scan_kernel(DevState* st, const __half* __restrict__ pooled,
                                                         const __half* __restrict__ q_idx,
                                                         const float* __restrict__ w,
                                                         float* __restrict__ scores, float rope_base) {
  constexpr int VPL = D / 32;  // dims per lane
  constexpr int U = 4;         // blocks in flight per warp
  __shared__ float s_q[H][D];
  __shared__ float s_cos[D / 2], s_sin[D / 2];

  pdl_wait();
  const int n = ld_volatile(&st->n_ctx);
  const int n_blocks = n / kBlock;
  if (ld_volatile(&st->n_pooled) != n_blocks) {
    if (blockIdx.x == 0 && threadIdx.x == 0) record_status(st, QSA_ERR_STATE);
    return;
  }
  // RoPE of the query at position n-1 (angles in double, rotation in f32)
  for (int i = threadIdx.x; i < D / 2; i += blockDim.x) {
    const double theta = pow((double)rope_base, -2.0 * (double)i / (double)D);
    double sd, cd;
    sincos((double)(n - 1) * theta, &sd, &cd);
    s_cos[i] = (float)cd;
    s_sin[i] = (float)sd;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < H * (D / 2); e += blockDim.x) {
    const int h = e / (D / 2), i = e % (D / 2);
    const float x1 = __half2float(q_idx[h * D + i]);
    const float x2 = __half2float(q_idx[h * D + i + D / 2]);
    s_q[h][i] = x1 * s_cos[i] - x2 * s_sin[i];
    s_q[h][i + D / 2] = x1 * s_sin[i] + x2 * s_cos[i];
  }
  __syncthreads();

  const int lane = threadIdx.x & 31;
  float qr[H][VPL];
#pragma unroll
  for (int h = 0; h < H; ++h)
#pragma unroll
    for (int j = 0; j < VPL; ++j) qr[h][j] = s_q[h][lane * VPL + j];
  const int my_head = head_of_lane<H>(lane);
  const float w_mine = w[my_head];
  const float sqrt_d = sqrtf((float)D);

  const int warps = blockDim.x >> 5;
  const int gw = blockIdx.x * warps + (threadIdx.x >> 5);
  const int total_warps = gridDim.x * warps;
  for (int b0 = gw * U; b0 < n_blocks; b0 += total_warps * U) {
    float p[U][VPL];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int b = b0 + u;
      if (b < n_blocks) {
        const __half* row = pooled + size_t(b) * D + lane * VPL;
        if constexpr (VPL == 4) {
          const uint2 raw = *reinterpret_cast<const uint2*>(row);
          const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
          const float2 c = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
          p[u][0] = a.x; p[u][1] = a.y; p[u][2] = c.x; p[u][3] = c.y;
        } else {
          const float2 a = __half22float2(*reinterpret_cast<const __half2*>(row));
          p[u][0] = a.x; p[u][1] = a.y;
        }
      } else {
#pragma unroll
        for (int j = 0; j < VPL; ++j) p[u][j] = 0.0f;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float dot[H];
#pragma unroll
      for (int h = 0; h < H; ++h) {
        float acc = 0.0f;
#pragma unroll
        for (int j = 0; j < VPL; ++j) acc = fmaf(qr[h][j], p[u][j], acc);
        dot[h] = acc;
      }
      const float mine = transpose_reduce<H>(dot, lane);
      const float total = sum_over_heads<H>(w_mine * fmaxf(mine, 0.0f));
      const int b = b0 + u;
      if (lane == 0 && b < n_blocks) scores[b] = total / sqrt_d;
    }
  }
}

template <int D>
static cudaError_t launch_scan_d(const LayerView& L, const void* q_idx, const float* w, float* scores,
                                 cudaStream_t s) {
  const dim3 grid(L.n_sms * 2), block(256);
  const float base = L.cfg.rope_base;
  switch (L.cfg.n_idx_heads) {
    case 1: return launch_pdl(index_scan_kernel<D, 1>, grid, block, 0, s, 1, L.state, (const __half*)L.pooled_cache, (const __half*)q_idx, w, scores, base);
    case 2: return launch_pdl(index_scan_kernel<D, 2>, grid, block, 0, s, 1, L.state, (const __half*)L.pooled_cache, (const __half*)q_idx, w, scores, base);
    case 4: return launch_pdl(index_scan_kernel<D, 4>, grid, block, 0, s, 1, L.state, (const __half*)L.pooled_cache, (const __half*)q_idx, w, scores, base);
    case 8: return launch_pdl(index_scan_kernel<D, 8>, grid, block, 0, s, 1, L.state, (const __half*)L.pooled_cache, (const __half*)q_idx, w, scores, base);
    case 16: return launch_pdl(index_scan_kernel<D, 16>, grid, block, 0, s, 1, L.state, (const __half*)L.pooled_cache, (const __half*)q_idx, w, scores, base);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_index_scan(const LayerView& L, const void* q_idx, const float* w, float* scores,
                              cudaStream_t s) {
  return L.cfg.d_idx == 128 ? launch_scan_d<128>(L, q_idx, w, scores, s)
                            : launch_scan_d<64>(L, q_idx, w, scores, s);
}

// ---------------------------------------------------------------------------------
// Block top-k: one cluster of kTopkCluster CTAs runs an exact radix select on 32-bit
// order-preserving keys of the scores (4 passes of 8 bits, stopping early once every
// key with the current prefix is needed). Histograms are merged through distributed
// shared memory. Ties at the threshold are taken in ascending block order, and the
// output is written in ascending block order (CTA r owns a contiguous index range).
// ---------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t score_key(float s) {
  if (s != s) return 0u;                        // NaN ranks lowest
  uint32_t u = __float_as_uint(s);
  if ((u & 0x7fffffffu) == 0u) u = 0u;          // -0 and +0 are the same score
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix sum of one value per thread over the whole CTA (blockDim == 1024).
// Returns the exclusive prefix; *total receives the CTA total.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* s_warp, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  __syncthreads();  // s_warp may still be read by a previous scan
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t t = s_warp[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, t, off);
      if (lane >= off) t += y;
    }
    s_warp[lane] = t;  // inclusive prefix of warp totals
  }
  __syncthreads();
  *total = s_warp[31];
  return (warp ? s_warp[warp - 1] : 0u) + x - v;
}

__global__ void __launch_bounds__(kTopkThreads, 1) block_topk_kernel(DevState* st, const float* __restrict__ scores,
                                                                       int32_t* __restrict__ sel,
                                                                       int32_t* __restrict__ n_sel, int k_blocks) {
  extern __shared__ uint32_t s_keys[];
  __shared__ uint32_t s_hist[2][256];
  __shared__ uint32_t s_warp[32];
  __shared__ uint32_t s_ctl[4];   // digit, count above digit, count at digit
  __shared__ uint32_t s_cta[2];   // this CTA's (greater, equal) counts, read by the cluster

  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int tid = threadIdx.x;

  pdl_wait();
  const int n = ld_volatile(&st->n_ctx);
  const int n_blocks = n / kBlock;
  if (ld_volatile(&st->n_pooled) != n_blocks) {
    if (rank == 0 && tid == 0) {
      record_status(st, QSA_ERR_STATE);
      *n_sel = 0;
    }
    return;  // uniform over the cluster: no shared memory of another CTA is touched
  }
  if (n_blocks <= k_blocks) {  // every block is selected
    for (int i = rank * blockDim.x + tid; i < n_blocks; i += C * blockDim.x) sel[i] = i;
    if (rank == 0 && tid == 0) *n_sel = n_blocks;
    return;
  }
  const int chunk = (n_blocks + C - 1) / C;
  const int start = rank * chunk;
  const int cnt = max(0, min(chunk, n_blocks - start));
  for (int j = tid; j < cnt; j += blockDim.x) s_keys[j] = score_key(scores[start + j]);
  __syncthreads();

  uint32_t prefix = 0, mask = 0;
  uint32_t need = (uint32_t)k_blocks;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    uint32_t* hist = s_hist[pass & 1];
    if (tid < 256) hist[tid] = 0;
    __syncthreads();
    for (int j = tid; j < cnt; j += blockDim.x) {
      const uint32_t key = s_keys[j];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    cluster.sync();
    // bins of the whole cluster; thread t < 256 holds bin (255 - t) so that an inclusive
    // prefix over t is the count of keys with digit >= 255 - t
    uint32_t v = 0;
    if (tid < 256) {
      const int bin = 255 - tid;
      for (int r = 0; r < C; ++r) v += cluster.map_shared_rank(hist, r)[bin];
    }
    uint32_t total;
    const uint32_t excl = block_exclusive_scan(tid < 256 ? v : 0u, s_warp, &total);
    if (tid < 256) {
      const uint32_t ge = excl + v;  // keys with digit >= bin
      if (ge >= need && excl < need) {
        s_ctl[0] = 255 - tid;
        s_ctl[1] = excl;
        s_ctl[2] = v;
      }
    }
    __syncthreads();
    const uint32_t digit = s_ctl[0];
    need -= s_ctl[1];
    prefix |= digit << shift;
    mask |= 255u << shift;
    const uint32_t at_digit = s_ctl[2];
    __syncthreads();
    if (at_digit == need) break;  // all keys with this prefix are selected
  }

  // Classify: greater than the threshold prefix, or equal to it (ties by block order).
  const int per = (cnt + blockDim.x - 1) / blockDim.x;
  const int j0 = tid * per, j1 = min(cnt, j0 + per);
  uint32_t c_gt = 0, c_eq = 0;
  for (int j = j0; j < j1; ++j) {
    const uint32_t km = s_keys[j] & mask;
    c_gt += km > prefix;
    c_eq += km == prefix;
  }
  uint32_t eq_total, gt_total;
  const uint32_t eq_before_thread = block_exclusive_scan(c_eq, s_warp, &eq_total);
  block_exclusive_scan(c_gt, s_warp, &gt_total);
  if (tid == 0) {
    s_cta[0] = gt_total;
    s_cta[1] = eq_total;
  }
  cluster.sync();
  uint32_t eq_before_cta = 0, out_before_cta = 0;
  for (int r = 0; r < rank; ++r) {
    const uint32_t* o = cluster.map_shared_rank(s_cta, r);
    const uint32_t g = o[0], e = o[1];
    const uint32_t taken = need > eq_before_cta ? min(e, need - eq_before_cta) : 0u;
    out_before_cta += g + taken;
    eq_before_cta += e;
  }
  const uint32_t rank0 = eq_before_cta + eq_before_thread;  // global tie rank of my first tie
  const uint32_t my_taken = need > rank0 ? min(c_eq, need - rank0) : 0u;
  uint32_t out_total;
  uint32_t pos = out_before_cta + block_exclusive_scan(c_gt + my_taken, s_warp, &out_total);
  uint32_t tie_rank = rank0;
  for (int j = j0; j < j1; ++j) {
    const uint32_t km = s_keys[j] & mask;
    bool take = km > prefix;
    if (km == prefix) take = tie_rank++ < need;
    if (take) sel[pos++] = start + j;
  }
  if (rank == 0 && tid == 0) *n_sel = k_blocks;
  cluster.sync();  // keep this CTA's shared memory alive until every remote read is done
}

cudaError_t init_kernel_attributes() {
  // shared-memory opt-in of the top-k cluster (set once per process and device, before
  // any launch, so that no attribute call happens while a stream is being captured)
  return cudaFuncSetAttribute(block_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kTopkMaxPerCta * (int)sizeof(uint32_t));
}

cudaError_t launch_topk(const LayerView& L, const float* scores, int32_t* sel, int32_t* n_sel, cudaStream_t s) {
  const int max_blocks = L.cfg.max_ctx / kBlock;
  const int chunk = (max_blocks + kTopkCluster - 1) / kTopkCluster;
  const size_t smem = size_t(chunk) * sizeof(uint32_t);
  return launch_pdl(block_topk_kernel, dim3(kTopkCluster), dim3(kTopkThreads), smem, s, kTopkCluster,
                    L.state, scores, sel, n_sel, L.cfg.top_k_tokens / kBlock);
}

}  // namespace qsa
