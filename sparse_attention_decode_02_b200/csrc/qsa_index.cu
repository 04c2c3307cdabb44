// Block-domain top-k (the indexer scan that produces the scores is in qsa_scan_tc.cu).
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
