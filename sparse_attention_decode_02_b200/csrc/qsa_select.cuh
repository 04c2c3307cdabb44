// Block-domain top-k as a device routine run by one cluster of kTopkCluster CTAs of
// kTopkThreads threads (used by the selection kernel in qsa_index.cu).
//
// Web page "Part 10" (第10回 EVO-X2 ... 長コンテキストのTGを高速化した話):
//  - section "QSA indexer": the high-scoring blocks are chosen by top-k;
//  - section "block-domain top-k（COMMON-006）実装は見送り": select in the block domain,
//    then expand only the chosen blocks into cells (never every cell of the context).
// Rule of this library: the min(K, B) largest scores, ties to the lower block index,
// output in ascending block order.
//
// An exact radix select on order-preserving 32-bit keys: 8-bit digits from the top,
// stopping as soon as every key with the current prefix is needed. CTA r of the cluster
// owns blocks [r*kTopkThreads*V, (r+1)*kTopkThreads*V), thread t the V consecutive blocks
// starting at t*V, held in registers. Per pass, each CTA histograms its keys in shared
// memory and pushes the histogram into every CTA's inbox with distributed-shared-memory
// stores; after one cluster barrier each CTA adds the histograms from its own memory. The
// output position of a selected block is the number of keys above the threshold before
// it plus min(need, ties before it), so one packed prefix scan and one pushed exchange of
// per-CTA totals give every position; ties are taken in block order. No CTA reads
// another's shared memory.
#pragma once

#include <cooperative_groups.h>

#include "qsa_device.cuh"

namespace qsa {

namespace sel {

namespace cg = cooperative_groups;

constexpr int kThreads = kTopkThreads;
constexpr int kCS = kTopkCluster;

// Order-preserving 32-bit key of a score: larger score <=> larger key.
__device__ __forceinline__ uint32_t score_key(float s) {
  if (s != s) return 0u;                        // NaN ranks lowest
  uint32_t u = __float_as_uint(s);
  if ((u & 0x7fffffffu) == 0u) u = 0u;          // -0 and +0 are the same score
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix sum of one value per thread over the CTA (kThreads threads, fixed
// order); *total receives the CTA total. s_warp holds 32 words.
__device__ __forceinline__ uint32_t cta_exclusive_scan(uint32_t v, uint32_t* s_warp, uint32_t* total) {
  constexpr int W = kThreads / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  __syncthreads();  // the previous user of s_warp is done
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {  // exclusive scan of the warp totals, one shuffle pass
    const uint32_t t = lane < W ? s_warp[lane] : 0u;
    uint32_t y = t;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t z = __shfl_up_sync(0xffffffffu, y, off);
      if (lane >= off) y += z;
    }
    if (lane < W) s_warp[lane] = y - t;
    if (lane == W - 1) s_warp[31] = y;
  }
  __syncthreads();
  *total = s_warp[31];
  return s_warp[warp] + x - v;
}

enum { kStale = 0, kAll = 1, kTopK = 2 };

struct Result {
  int status;    // kStale: pooled cache behind the context (nothing selected)
                 // kAll: n_blocks <= K, every block is selected (emit not called)
                 // kTopK: K blocks emitted
  int n_ctx;
  int n_blocks;
};

// Preconditions: every thread of the cluster executed cluster_arrive_relaxed() and then
// pdl_wait(). Selects among the blocks completed within the first n_ctx - n_back tokens
// (n_back > 0: a query of an earlier token of a multi-query step). Calls
// emit(position, block) once per selected block (kTopK only) and returns the same result
// in every thread of the cluster. Cluster-barrier pairing is complete on return on every
// path.
template <int V, class Emit>
__device__ __forceinline__ Result cluster_select(DevState* st, const float* __restrict__ scores, int k_blocks,
                                                 int max_blocks, int n_back, Emit&& emit) {
  __shared__ uint32_t s_hist[256];          // this CTA's histogram of the pass
  __shared__ uint32_t s_in[2][kCS][256];    // every CTA's histogram, double-buffered by pass
  __shared__ uint32_t s_warp[32];
  __shared__ uint32_t s_ctl[4];             // digit, count above the digit, count at the digit
  __shared__ uint32_t s_all[2 * kCS];       // every CTA's (greater, equal) totals

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = int(cluster.block_rank());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // this thread's V scores, read up to the buffer's capacity (max_ctx/4) in the same round
  // trip as the state; blocks at or past n_ctx/4 are masked once the state is known
  const int base = rank * kThreads * V + tid * V;
  float f[V];
  if (base + V <= max_blocks) {
#pragma unroll
    for (int j = 0; j < V; j += 4) {
      const float4 x = *reinterpret_cast<const float4*>(scores + base + j);
      f[j] = x.x;
      f[j + 1] = x.y;
      f[j + 2] = x.z;
      f[j + 3] = x.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < V; ++j) f[j] = base + j < max_blocks ? scores[base + j] : 0.0f;
  }
  const int n_full = ld_volatile(&st->n_ctx);
  const int n_pooled = ld_volatile(&st->n_pooled);
#pragma unroll
  for (int j = 0; j < V; ++j) asm volatile("" ::"f"(f[j]));  // keep the loads ahead of the branches
  const int n = n_full - n_back;
  const int n_blocks = n / kBlock;
  if (n_pooled != n_full / kBlock || n < 0) {  // uniform over the cluster
    if (rank == 0 && tid == 0) record_status(st, QSA_ERR_STATE);
    cluster_wait();
    return Result{kStale, n, 0};
  }
  if (n_blocks <= k_blocks) {  // uniform over the cluster
    cluster_wait();
    return Result{kAll, n, n_blocks};
  }

  uint32_t key[V];
  uint32_t valid = 0;  // bit j: block base + j exists
#pragma unroll
  for (int j = 0; j < V; ++j) {
    key[j] = score_key(f[j]);
    if (base + j < n_blocks) valid |= 1u << j;
  }
  if (tid < 256) s_hist[tid] = 0;
  cluster_wait();  // every CTA of the cluster has started: its shared memory may be written

  uint32_t prefix = 0, mask = 0, need = uint32_t(k_blocks);
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    __syncthreads();  // the local histogram is zeroed
#pragma unroll
    for (int j = 0; j < V; ++j)
      if (((valid >> j) & 1u) && (key[j] & mask) == prefix) atomicAdd(&s_hist[(key[j] >> shift) & 255u], 1u);
    __syncthreads();
    // push bin t into slot [rank][t] of every CTA's inbox for this pass, and clear it for
    // the next pass. A CTA reuses an inbox buffer two passes later, after a barrier that
    // every CTA passes only once all have finished reading it.
    if (tid < 256) {
      const uint32_t mine = s_hist[tid];
      s_hist[tid] = 0;
#pragma unroll
      for (int r = 0; r < kCS; ++r) cluster.map_shared_rank(&s_in[pass & 1][0][0], r)[rank * 256 + tid] = mine;
    }
    cluster.sync();  // release the pushes, acquire every other CTA's
    // thread t < 256 takes digit (255 - t): an inclusive prefix over t counts keys >= digit
    uint32_t v = 0;
    if (tid < 256) {
      const int bin = 255 - tid;
#pragma unroll
      for (int r = 0; r < kCS; ++r) v += s_in[pass & 1][r][bin];
    }
    uint32_t x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    if (lane == 31 && warp < 8) s_warp[warp] = x;
    __syncthreads();
    if (tid < 256) {
      uint32_t excl = x - v;
#pragma unroll
      for (int w = 0; w < 8; ++w) excl += w < warp ? s_warp[w] : 0u;
      if (excl < need && excl + v >= need) {
        s_ctl[0] = uint32_t(255 - tid);
        s_ctl[1] = excl;
        s_ctl[2] = v;
      }
    }
    __syncthreads();
    need -= s_ctl[1];
    prefix |= s_ctl[0] << shift;
    mask |= 255u << shift;
    if (s_ctl[2] == need) break;  // every key with this prefix is selected (uniform)
  }

  // classify: above the threshold prefix, or equal to it (ties go by block order)
  uint32_t c_gt = 0, c_eq = 0;
#pragma unroll
  for (int j = 0; j < V; ++j) {
    if (!((valid >> j) & 1u)) continue;
    const uint32_t km = key[j] & mask;
    c_gt += km > prefix;
    c_eq += km == prefix;
  }
  uint32_t tot;
  const uint32_t before = cta_exclusive_scan((c_gt << 16) | c_eq, s_warp, &tot);
  if (tid < kCS) {  // push this CTA's totals to every CTA
    uint32_t* dst = cluster.map_shared_rank(s_all, tid);
    dst[2 * rank] = tot >> 16;
    dst[2 * rank + 1] = tot & 0xffffu;
  }
  cluster.sync();
  uint32_t gt_before = before >> 16, eq_before = before & 0xffffu;
#pragma unroll
  for (int r = 0; r < kCS; ++r) {
    gt_before += r < rank ? s_all[2 * r] : 0u;
    eq_before += r < rank ? s_all[2 * r + 1] : 0u;
  }
#pragma unroll
  for (int j = 0; j < V; ++j) {
    if (!((valid >> j) & 1u)) continue;
    const uint32_t km = key[j] & mask;
    if (km > prefix) {
      emit(gt_before + min(need, eq_before), base + j);
      ++gt_before;
    } else if (km == prefix) {
      if (eq_before < need) emit(gt_before + eq_before, base + j);
      ++eq_before;
    }
  }
  return Result{kTopK, n, n_blocks};
}

// Keys each thread holds for a layer of max_blocks blocks: 8, 16 or 32.
inline int keys_per_thread(int max_blocks) {
  return max_blocks <= kCS * kThreads * 8 ? 8 : max_blocks <= kCS * kThreads * 16 ? 16 : 32;
}

}  // namespace sel
}  // namespace qsa
