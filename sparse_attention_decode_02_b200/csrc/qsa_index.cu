// Block-domain top-k (the indexer scan that produces the scores is in qsa_scan_tc.cu).
//
// Web page "Part 10" (第10回 EVO-X2 ... 長コンテキストのTGを高速化した話):
//  - section "QSA indexer": the high-scoring blocks are chosen by top-k;
//  - section "block-domain top-k（COMMON-006）実装は見送り": select in the block domain,
//    then expand only the chosen blocks into cells (never every cell of the context).
// Rule of this library: the min(K, B) largest scores, ties to the lower block index,
// output in ascending block order.
#include <cooperative_groups.h>
#include <cuda_fp16.h>

#include "qsa_select.cuh"
#include "qsa_checked.cuh"
#include "qsa_timeline.cuh"

namespace qsa {

// Stand-alone selection: one cluster runs the radix select of qsa_select.cuh and writes
// the selected blocks in ascending order. With gridDim.y = T > 1 (multi-query step),
// cluster u selects for the query of token n_ctx - T + u from score row u into output
// row u (rows of k_blocks ids, one count each).
// With `hist`, cluster u starts from query u's score-key histogram (hist + u * 2048).
// With sel_scores (single query): a context-parallel shard's candidate slots, below.
template <int V>
__global__ void __launch_bounds__(sel::kThreads, 1)
block_topk_kernel(DevState* st, const float* __restrict__ scores, int32_t* __restrict__ sel_out,
                  int32_t* __restrict__ n_sel, int k_blocks, int max_blocks, int score_stride, uint32_t* hist,
                  float* __restrict__ sel_scores, int block_base, int fused_max_ctx) {
  const int rank = int(cooperative_groups::this_cluster().block_rank());
  const int u = blockIdx.y, n_back = gridDim.y - 1 - blockIdx.y;
  scores += size_t(u) * score_stride;
  sel_out += size_t(u) * k_blocks;
  n_sel += u;
  __shared__ uint64_t s_gather_bar;  // CTA 0: every CTA's candidates have landed (histogram path)
  if (threadIdx.x == 0) {
    sm100::mbar_init(&s_gather_bar, sel::kCS);
    sm100::fence_mbar_init();
  }
  pdl_launch_dependents();
  if (threadIdx.x == 0) QSA_TL(st, kTlTopk, kTlEntry);
  cluster_arrive_relaxed();  // paired inside cluster_select
  pdl_wait();
  if (threadIdx.x == 0) QSA_TL(st, kTlTopk, kTlWait);
  // query u's histogram (the multi-query scan fills one per query)
  const sel::Result res = sel::cluster_select<V>(st, scores, hist ? hist + size_t(u) * (1u << kHistBits) : nullptr,
                                                 k_blocks, max_blocks,
                                                 n_back, &s_gather_bar, gridDim.y == 1 ? fused_max_ctx : 0,
                                                 [&](uint32_t pos, int block) {
                                                   // bounds-checked in every build
                                                   if (pos < uint32_t(k_blocks) && block < max_blocks) {
                                                     sel_out[pos] = block + block_base;
                                                     if (sel_scores) sel_scores[pos] = scores[block];
                                                   } else {
                                                     record_status(st, QSA_ERR_BAD_INDEX);
                                                   }
                                                 });
  if (res.status == sel::kAll)
    for (int i = rank * sel::kThreads + threadIdx.x; i < res.n_blocks; i += sel::kCS * sel::kThreads) {
      sel_out[i] = i + block_base;
      if (sel_scores) sel_scores[i] = scores[i];
    }
  const int count = res.status == sel::kTopK ? k_blocks : res.status == sel::kAll ? res.n_blocks : 0;
  if (rank == 0 && threadIdx.x == 0) *n_sel = count;
  // candidate slots: the positions past the count hold score -inf and block -1
  if (sel_scores)
    for (int i = rank * sel::kThreads + threadIdx.x; i < k_blocks; i += sel::kCS * sel::kThreads)
      if (i >= count) {
        sel_scores[i] = -INFINITY;
        sel_out[i] = -1;
      }
  if (threadIdx.x == 0) QSA_TL(st, kTlTopk, kTlExit);
}

namespace {
template <int V>
cudaError_t set_topk_attr() {
  cudaError_t e = cudaFuncSetAttribute(block_topk_kernel<V>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(block_topk_kernel<V>, cudaFuncAttributePreferredSharedMemoryCarveout, kCarveoutMaxShared);
  return e;
}
}  // namespace

cudaError_t init_kernel_attributes() {
  cudaError_t e;
  if ((e = set_topk_attr<8>()) != cudaSuccess || (e = set_topk_attr<16>()) != cudaSuccess ||
      (e = set_topk_attr<32>()) != cudaSuccess)
    return e;
  // the cluster needs kCS SMs of one GPC at once: check that the device can host it
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sel::kCS);
  cfg.blockDim = dim3(sel::kThreads);
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = sel::kCS;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int active = 0;
  if ((e = cudaOccupancyMaxActiveClusters(&active, block_topk_kernel<32>, &cfg)) != cudaSuccess) return e;
  return active >= 1 ? cudaSuccess : cudaErrorNotSupported;
}

cudaError_t launch_topk(const LayerView& L, const float* scores, int32_t* sel_out, int32_t* n_sel, cudaStream_t s,
                        int n_queries, int score_stride, uint32_t* hist, float* sel_scores, int block_base,
                        bool after_fused_scan) {
  if (n_queries != 1) sel_scores = nullptr, block_base = 0, after_fused_scan = false;
  const int max_blocks = L.cfg.max_ctx / kBlock;
  const int kb = L.cfg.top_k_tokens / kBlock;
  const int fused_max_ctx = after_fused_scan ? L.cfg.max_ctx : 0;
  const dim3 grid(sel::kCS, n_queries), block(sel::kThreads);
  if (max_blocks <= sel::kCS * sel::kThreads * 8)
    return launch_pdl(block_topk_kernel<8>, grid, block, 0, s, sel::kCS, L.state, scores, sel_out, n_sel, kb,
                      max_blocks, score_stride, hist, sel_scores, block_base, fused_max_ctx);
  if (max_blocks <= sel::kCS * sel::kThreads * 16)
    return launch_pdl(block_topk_kernel<16>, grid, block, 0, s, sel::kCS, L.state, scores, sel_out, n_sel, kb,
                      max_blocks, score_stride, hist, sel_scores, block_base, fused_max_ctx);
  return launch_pdl(block_topk_kernel<32>, grid, block, 0, s, sel::kCS, L.state, scores, sel_out, n_sel, kb,
                    max_blocks, score_stride, hist, sel_scores, block_base, fused_max_ctx);
}

}  // namespace qsa
