// Context-parallel form of one decode step: the context of one layer is split into
// contiguous, block-aligned shards, one per device (the last holding the open tail).
//
// Web page "Part 10" (第10回 EVO-X2 ... 長コンテキストのTGを高速化した話), section "QSAと
// QSA indexerについて": long context is handled by sparsity, the selected set being small
// whatever the context length; a context beyond one device's memory is sharded here. The
// step is exact: every block of the global top-K is in its own shard's local top-K (fewer
// than K blocks beat it anywhere), and candidates listed shard by shard in ascending block
// order keep "ties to the lower block" intact, so the merged selection and the merged
// attention equal the single-device step.
//
// Kernels here (the shard's scan and local top-K reuse qsa_scan_tc.cu and qsa_index.cu):
//  - cp_select_kernel: the global top-K of every shard's candidate slots (one CTA);
//  - cp_filter_kernel: the part of the global selection that falls in this shard's blocks,
//    as local block ids (ascending), for the shard's attention;
//  - cp_merge_kernel: the exact merge of per-shard attention partials,
//    o = sum_r exp(lse_r - LSE) o_r / sum_r exp(lse_r - LSE).
#include <cuda_fp16.h>

#include "qsa_device.cuh"
#include "qsa_select.cuh"

namespace qsa {

namespace {

constexpr int kCpThreads = 1024;
constexpr int kCpPer = 8;  // candidate slots per thread: shards * K <= 8192

// Exclusive prefix sum over the CTA in thread order; *total gets the CTA total.
__device__ __forceinline__ uint32_t cp_exclusive_scan(uint32_t v, uint32_t* s_warp, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  __syncthreads();
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const uint32_t t = lane < nw ? s_warp[lane] : 0u;
    uint32_t y = t;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t z = __shfl_up_sync(0xffffffffu, y, off);
      if (lane >= off) y += z;
    }
    if (lane < nw) s_warp[lane] = y - t;
    if (lane == 31) s_warp[32] = y;
  }
  __syncthreads();
  *total = s_warp[32];
  return s_warp[warp] + x - v;
}

}  // namespace

// The global top-K of n_slots = shards * K candidate slots (scores, global block ids; a slot
// with block id -1 is empty), listed shard by shard, each shard's in ascending block order.
// Rule: the K largest scores, ties to the lower block, output ascending; fewer than K
// candidates: all of them. Thread t holds slots [8t, 8t + 8), so slot order is thread order;
// T threads take up to 8T slots (T = 256 up to 2048 slots: the CTA-wide barriers and
// scans of a smaller CTA are cheaper). A 2048-bin histogram of the keys' top 11 bits gives
// the bin of the K-th key; radix passes over the remaining 21 bits (8, 8, 5) refine inside
// it, warp 0 scanning each pass's digit counts; one packed prefix scan places every
// selected slot.
template <int T>
__global__ void __launch_bounds__(T) cp_select_kernel(const float* __restrict__ cand_scores,
                                                      const int32_t* __restrict__ cand_blocks, int n_slots,
                                                      int k_blocks, int32_t* __restrict__ sel,
                                                      int32_t* __restrict__ n_sel) {
  constexpr int kHB = 2048;
  constexpr int kBinsPer = kHB / T;  // histogram bins per thread, from the top
  static_assert(kBinsPer * T == kHB && T >= 256, "whole bins per thread; 256 digit bins per pass");
  __shared__ uint32_t s_h[kHB];
  __shared__ uint32_t s_warp[33];
  __shared__ uint32_t s_ctl[4];
  const int tid = threadIdx.x, base = tid * kCpPer, lane = tid & 31, warp = tid >> 5;
  pdl_launch_dependents();
  pdl_wait();
  uint32_t key[kCpPer];
  int32_t blk[kCpPer];
  uint32_t valid = 0;
#pragma unroll
  for (int j = 0; j < kCpPer; ++j) {
    const int i = base + j;
    blk[j] = i < n_slots ? cand_blocks[i] : -1;
    key[j] = i < n_slots ? sel::score_key(cand_scores[i]) : 0u;
    if (blk[j] >= 0) valid |= 1u << j;
  }
  for (int i = tid; i < kHB; i += T) s_h[i] = 0u;
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kCpPer; ++j)
    if ((valid >> j) & 1u) atomicAdd(&s_h[key[j] >> 21], 1u);
  __syncthreads();
  // thread t holds bins 2047 - kBinsPer*t - q, q < kBinsPer (from the top); keys above
  // them come first
  uint32_t hb[kBinsPer], hsum = 0;
#pragma unroll
  for (int q = 0; q < kBinsPer; ++q) {
    hb[q] = s_h[kHB - 1 - kBinsPer * tid - q];
    hsum += hb[q];
  }
  uint32_t total;
  const uint32_t above = cp_exclusive_scan(hsum, s_warp, &total);
  uint32_t prefix = 0, mask = 0, need = uint32_t(k_blocks);
  const bool all = total <= uint32_t(k_blocks);  // uniform
  if (all) {
    need = total;  // mask 0: every valid slot is "at the threshold" and taken
  } else {
    uint32_t acc = above;
#pragma unroll
    for (int q = 0; q < kBinsPer; ++q) {
      if (acc < need && acc + hb[q] >= need) {
        s_ctl[0] = uint32_t(kHB - 1 - kBinsPer * tid - q);
        s_ctl[1] = acc;
      }
      acc += hb[q];
    }
    __syncthreads();
    prefix = s_ctl[0] << 21;
    mask = ~0u << 21;
    need -= s_ctl[1];
    __syncthreads();  // s_ctl is rewritten below
    for (int shift = 13;; shift -= 8) {  // bits 20..13, 12..5, 4..0
      const int bits = shift >= 0 ? 8 : 8 + shift;
      shift = shift >= 0 ? shift : 0;
      const uint32_t nb = 1u << bits;
      if (tid < 256) s_h[tid] = 0u;
      __syncthreads();
#pragma unroll
      for (int j = 0; j < kCpPer; ++j)
        if (((valid >> j) & 1u) && (key[j] & mask) == prefix) atomicAdd(&s_h[(key[j] >> shift) & (nb - 1)], 1u);
      __syncthreads();
      if (warp == 0) {  // lane l: digits nb-1-8l .. nb-8-8l (from the top)
        uint32_t cq[8], sum = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int d = int(nb) - 1 - (8 * lane + q);
          cq[q] = d >= 0 ? s_h[d] : 0u;
          sum += cq[q];
        }
        uint32_t x = sum;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, x, off);
          if (lane >= off) x += y;
        }
        uint32_t acc = x - sum;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (acc < need && acc + cq[q] >= need) {
            s_ctl[0] = nb - 1 - uint32_t(8 * lane + q);
            s_ctl[1] = acc;
            s_ctl[2] = cq[q];
          }
          acc += cq[q];
        }
      }
      __syncthreads();
      need -= s_ctl[1];
      prefix |= s_ctl[0] << shift;
      mask |= (nb - 1) << shift;
      const bool done = s_ctl[2] == need || shift == 0;
      __syncthreads();  // s_ctl and s_h are rewritten by the next pass
      if (done) break;
    }
  }
  // positions: keys above the threshold before this one, plus min(need, ties before it)
  uint32_t c_gt = 0, c_eq = 0;
#pragma unroll
  for (int j = 0; j < kCpPer; ++j) {
    if (!((valid >> j) & 1u)) continue;
    const uint32_t km = key[j] & mask;
    c_gt += km > prefix;
    c_eq += km == prefix;
  }
  uint32_t tot;
  const uint32_t before = cp_exclusive_scan((c_gt << 16) | c_eq, s_warp, &tot);
  uint32_t gt_b = before >> 16, eq_b = before & 0xffffu;
#pragma unroll
  for (int j = 0; j < kCpPer; ++j) {
    if (!((valid >> j) & 1u)) continue;
    const uint32_t km = key[j] & mask;
    if (km > prefix) {
      const uint32_t pos = gt_b + min(need, eq_b);
      if (pos < uint32_t(k_blocks)) sel[pos] = blk[j];
      ++gt_b;
    } else if (km == prefix) {
      if (eq_b < need && gt_b + eq_b < uint32_t(k_blocks)) sel[gt_b + eq_b] = blk[j];
      ++eq_b;
    }
  }
  if (tid == 0) *n_sel = int32_t(all ? total : uint32_t(k_blocks));
}

// The blocks of the global selection that belong to this shard ([block_base,
// block_base + n_ctx/4) of the global numbering), as local ids in ascending order, and
// their count; the shard's attention reads them like its own selection. The global
// selection is ascending and the shard's blocks contiguous, so its entries are one run of
// the list: an entry's position is its index less the count of entries below the shard.
__global__ void __launch_bounds__(kCpThreads) cp_filter_kernel(DevState* st, const int32_t* __restrict__ sel_global,
                                                               const int32_t* __restrict__ n_sel_global,
                                                               int block_base, int k_blocks,
                                                               int32_t* __restrict__ sel_local,
                                                               int32_t* __restrict__ n_local) {
  const int tid = threadIdx.x;
  pdl_launch_dependents();
  pdl_wait();
  const int nb = ld_volatile(&st->n_ctx) / kBlock;
  int ns = *n_sel_global;
  ns = ns < 0 ? 0 : (ns > k_blocks ? k_blocks : ns);
  int b = -1;
  bool keep = false, below = false;
  if (tid < ns) {
    b = sel_global[tid] - block_base;
    keep = b >= 0 && b < nb;
    below = b < 0;
  }
  const int lo = __syncthreads_count(below);
  const int total = __syncthreads_count(keep);
  if (keep && tid - lo < k_blocks) sel_local[tid - lo] = b;
  if (tid == 0) *n_local = total;
}

// out[i] = sum_r w_r o_r[i] / sum_r w_r, w_r = exp(lse_r[i] - max_r lse_r[i]) over the
// shards with a finite lse (an empty shard has lse -inf and weight 0); 0 if none.
__global__ void __launch_bounds__(128) cp_merge_kernel(const float* __restrict__ o_parts,
                                                       const float* __restrict__ lse_parts, int n_shards,
                                                       int n_q_heads, int head_dim, float* __restrict__ out) {
  pdl_launch_dependents();
  pdl_wait();
  const int i = blockIdx.x;
  float M = -INFINITY;
  for (int r = 0; r < n_shards; ++r) M = fmaxf(M, lse_parts[size_t(r) * n_q_heads + i]);
  for (int d = threadIdx.x; d < head_dim; d += blockDim.x) {
    float acc = 0.0f, den = 0.0f;
    if (M != -INFINITY) {
      for (int r = 0; r < n_shards; ++r) {
        const float l = lse_parts[size_t(r) * n_q_heads + i];
        if (l == -INFINITY) continue;
        const float e = expf(l - M);
        acc = fmaf(e, o_parts[(size_t(r) * n_q_heads + i) * head_dim + d], acc);
        den += e;
      }
    }
    out[size_t(i) * head_dim + d] = den > 0.0f ? acc / den : 0.0f;
  }
}

cudaError_t launch_cp_select(const float* cand_scores, const int32_t* cand_blocks, int n_shards, int k_blocks,
                             int32_t* sel, int32_t* n_sel, cudaStream_t s) {
  const int n_slots = n_shards * k_blocks;
  if (n_slots <= 256 * kCpPer)
    return launch_pdl(cp_select_kernel<256>, dim3(1), dim3(256), 0, s, 1, cand_scores, cand_blocks, n_slots,
                      k_blocks, sel, n_sel);
  return launch_pdl(cp_select_kernel<kCpThreads>, dim3(1), dim3(kCpThreads), 0, s, 1, cand_scores, cand_blocks,
                    n_slots, k_blocks, sel, n_sel);
}

cudaError_t launch_cp_filter(const LayerView& L, const int32_t* sel_global, const int32_t* n_sel_global,
                             int block_base, int32_t* sel_local, int32_t* n_local, cudaStream_t s) {
  // one thread per entry of the global selection (k_blocks <= kCpThreads)
  const int kb = L.cfg.top_k_tokens / kBlock;
  const int threads = kb >= kCpThreads ? kCpThreads : (kb + 31) / 32 * 32;
  return launch_pdl(cp_filter_kernel, dim3(1), dim3(threads), 0, s, 1, L.state, sel_global, n_sel_global,
                    block_base, L.cfg.top_k_tokens / kBlock, sel_local, n_local);
}

cudaError_t launch_cp_merge(const float* o_parts, const float* lse_parts, int n_shards, int n_q_heads, int head_dim,
                            float* out, cudaStream_t s) {
  return launch_pdl(cp_merge_kernel, dim3(n_q_heads), dim3(128), 0, s, 1, o_parts, lse_parts, n_shards, n_q_heads,
                    head_dim, out);
}

}  // namespace qsa
