// Selected K/V gather and GQA sparse attention.
//
// Web page "Part 10" (第10回 EVO-X2 ... 長コンテキストのTGを高速化した話):
//  - section "なぜFlash Attentionがcontext長に比例していたのか": with indexer_top_k = 2048
//    and compression ratio 4, at most 2048 + 4 - 1 = 2051 cells are attended (the
//    selected blocks plus the still-open tail block);
//  - section "selected QSA K/V gather（COMMON-005）": attend only over the selected rows
//    of K/V (the pages materialise compact K/V with get_rows and then run ordinary flash
//    attention). Here the gather is fused into a split-KV flash-decode kernel that reads
//    the selected rows straight from the f16 cache; qsa_gather_kv can still materialise
//    the compact K/V.
#include <cuda_fp16.h>

#include <cooperative_groups.h>

#include <mutex>

#include "qsa_device.cuh"

namespace cg = cooperative_groups;

namespace qsa {

// ---------------------------------------------------------------------------------
// Cell expansion: block b -> cells 4b..4b+3, then the open tail [4*(n/4), n).
// ---------------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) expand_cells_kernel(DevState* st, const int32_t* __restrict__ sel,
                                                            const int32_t* __restrict__ n_sel,
                                                            int32_t* __restrict__ cells,
                                                            int32_t* __restrict__ n_cells, int k_blocks) {
  pdl_wait();
  const int n = ld_volatile(&st->n_ctx);
  const int n_blocks = n / kBlock;
  int ns = *n_sel;
  if (ns < 0 || ns > k_blocks) {
    if (threadIdx.x == 0) record_status(st, QSA_ERR_BAD_INDEX);
    ns = ns < 0 ? 0 : k_blocks;
  }
  const int tail = n - kBlock * n_blocks;
  const int total = kBlock * ns + tail;
  for (int t = threadIdx.x; t < total; t += blockDim.x) {
    int cell;
    if (t < kBlock * ns) {
      const int b = sel[t / kBlock];
      if (b < 0 || b >= n_blocks) {
        record_status(st, QSA_ERR_BAD_INDEX);
        cell = -1;  // skipped by the attention kernel
      } else {
        cell = kBlock * b + (t % kBlock);
      }
    } else {
      cell = kBlock * n_blocks + (t - kBlock * ns);
    }
    cells[t] = cell;
  }
  if (threadIdx.x == 0) *n_cells = total;
}

// Literal compact K/V (the pages' get_rows(K), get_rows(V)): row c of k_out/v_out is
// the cache row of cells[c]; invalid cells give zero rows.
__global__ void __launch_bounds__(256) gather_rows_kernel(DevState* st, const int32_t* __restrict__ cells,
                                                          const int32_t* __restrict__ n_cells,
                                                          const uint4* __restrict__ kc, const uint4* __restrict__ vc,
                                                          uint4* __restrict__ k_out, uint4* __restrict__ v_out,
                                                          int row_units, int max_cells) {
  pdl_wait();
  const int n = ld_volatile(&st->n_ctx);
  int nc = *n_cells;
  nc = nc < 0 ? 0 : (nc > max_cells ? max_cells : nc);
  const size_t total = size_t(nc) * row_units;
  for (size_t e = size_t(blockIdx.x) * blockDim.x + threadIdx.x; e < total; e += size_t(gridDim.x) * blockDim.x) {
    const int c = int(e / row_units), u = int(e % row_units);
    const int cell = cells[c];
    uint4 kv = make_uint4(0, 0, 0, 0), vv = kv;
    if (cell >= 0 && cell < n) {
      kv = kc[size_t(cell) * row_units + u];
      vv = vc[size_t(cell) * row_units + u];
    }
    if (k_out) k_out[e] = kv;
    if (v_out) v_out[e] = vv;
  }
}

cudaError_t launch_gather(const LayerView& L, const int32_t* sel, const int32_t* n_sel, int32_t* cells,
                          int32_t* n_cells, void* k_compact, void* v_compact, cudaStream_t s) {
  cudaError_t e = launch_pdl(expand_cells_kernel, dim3(1), dim3(1024), 0, s, 1, L.state, sel, n_sel, cells,
                             n_cells, L.cfg.top_k_tokens / kBlock);
  if (e != cudaSuccess || (!k_compact && !v_compact)) return e;
  const int row_units = L.cfg.n_kv_heads * L.cfg.head_dim * 2 / 16;
  const int max_cells = max_cells_of(L.cfg);
  int grid = int((size_t(max_cells) * row_units + 255) / 256);
  if (grid > L.n_sms * 4) grid = L.n_sms * 4;
  return launch_pdl(gather_rows_kernel, dim3(grid), dim3(256), 0, s, 1, L.state, (const int32_t*)cells,
                    (const int32_t*)n_cells, (const uint4*)L.k_cache, (const uint4*)L.v_cache, (uint4*)k_compact,
                    (uint4*)v_compact, row_units, max_cells);
}

// ---------------------------------------------------------------------------------
// Split-KV flash decode with the gather fused in. CTA (split s, KV head g) takes cells
// [s*Lc, (s+1)*Lc) of the cell list; warp w takes every 8th of them. Lane l owns dims
// [l*VPL, (l+1)*VPL) of K, V and of the G query heads that share KV head g, so each
// warp reads every selected 2*D-byte K and V row of its cells with one coalesced load.
// Logits -> per-head max/sum over the CTA's cells (f32) -> unnormalised partial output
// with its (max, sum) pair; a second kernel merges the splits.
// ---------------------------------------------------------------------------------
template <int D, int G>
__global__ void __launch_bounds__(256) attn_split_kernel(DevState* st, const __half* __restrict__ q,
                                                         const int32_t* __restrict__ cells,
                                                         const int32_t* __restrict__ n_cells,
                                                         const __half* __restrict__ kc, const __half* __restrict__ vc,
                                                         float* __restrict__ part_o, float* __restrict__ part_ml,
                                                         int n_kv_heads, int cells_per_cta, int max_cells) {
  constexpr int VPL = D / 32;
  constexpr int W = kAttnWarps;
  constexpr int JMAX = kAttnMaxCells / W;
  constexpr int GR = G < 32 ? G : 32;  // heads reduced across lanes at once
  static_assert(G <= 8, "at most 8 query heads per KV head");
  __shared__ float s_p[G][kAttnMaxCells];
  __shared__ float s_o[W][G][D];
  __shared__ float s_m[G], s_l[G];

  const int split = blockIdx.x, g = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n_q_heads = n_kv_heads * G;

  pdl_wait();
  const int n = ld_volatile(&st->n_ctx);
  int nc = *n_cells;
  if (nc < 0 || nc > max_cells) {
    if (split == 0 && g == 0 && threadIdx.x == 0) record_status(st, QSA_ERR_BAD_INDEX);
    nc = nc < 0 ? 0 : max_cells;
  }
  const int c0 = split * cells_per_cta;
  const int my_cells = max(0, min(cells_per_cta, nc - c0));

  // this warp's cells: local index j*W + warp
  int cid[JMAX];
  bool valid[JMAX];
#pragma unroll
  for (int j = 0; j < JMAX; ++j) {
    const int lc = j * W + warp;
    cid[j] = lc < my_cells ? cells[c0 + lc] : -1;
    valid[j] = lc < my_cells && cid[j] >= 0 && cid[j] < n;
    if (lc < my_cells && !valid[j] && lane == 0) record_status(st, QSA_ERR_BAD_INDEX);
  }
  // issue every K and V row load before any arithmetic
  float kv_k[JMAX][VPL], kv_v[JMAX][VPL];
#pragma unroll
  for (int j = 0; j < JMAX; ++j) {
    if (valid[j]) {
      const size_t off = (size_t(cid[j]) * n_kv_heads + g) * D + lane * VPL;
      if constexpr (VPL == 4) {
        const uint2 rk = *reinterpret_cast<const uint2*>(kc + off);
        const uint2 rv = *reinterpret_cast<const uint2*>(vc + off);
        const float2 k0 = __half22float2(*reinterpret_cast<const __half2*>(&rk.x));
        const float2 k1 = __half22float2(*reinterpret_cast<const __half2*>(&rk.y));
        const float2 v0 = __half22float2(*reinterpret_cast<const __half2*>(&rv.x));
        const float2 v1 = __half22float2(*reinterpret_cast<const __half2*>(&rv.y));
        kv_k[j][0] = k0.x; kv_k[j][1] = k0.y; kv_k[j][2] = k1.x; kv_k[j][3] = k1.y;
        kv_v[j][0] = v0.x; kv_v[j][1] = v0.y; kv_v[j][2] = v1.x; kv_v[j][3] = v1.y;
      } else {
        const float2 k0 = __half22float2(*reinterpret_cast<const __half2*>(kc + off));
        const float2 v0 = __half22float2(*reinterpret_cast<const __half2*>(vc + off));
        kv_k[j][0] = k0.x; kv_k[j][1] = k0.y;
        kv_v[j][0] = v0.x; kv_v[j][1] = v0.y;
      }
    } else {
#pragma unroll
      for (int x = 0; x < VPL; ++x) kv_k[j][x] = kv_v[j][x] = 0.0f;
    }
  }
  float qv[G][VPL];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int x = 0; x < VPL; ++x) qv[h][x] = __half2float(q[(size_t(g) * G + h) * D + lane * VPL + x]);

  const float scale = 1.0f / sqrtf((float)D);
  // logits
#pragma unroll
  for (int j = 0; j < JMAX; ++j) {
    const int lc = j * W + warp;
    if (lc < my_cells) {  // warp-uniform
      float dot[GR];
#pragma unroll
      for (int h = 0; h < GR; ++h) {
        float a = 0.0f;
#pragma unroll
        for (int x = 0; x < VPL; ++x) a = fmaf(qv[h][x], kv_k[j][x], a);
        dot[h] = a;
      }
      const float mine = transpose_reduce<GR>(dot, lane);
      const int h = head_of_lane<GR>(lane);
      if ((lane & (32 / GR - 1)) == 0) s_p[h][lc] = valid[j] ? mine * scale : -INFINITY;
    }
  }
  __syncthreads();
  // per-head max and sum over this CTA's cells
  for (int h = warp; h < G; h += W) {
    float m = -INFINITY;
    for (int c = lane; c < my_cells; c += 32) m = fmaxf(m, s_p[h][c]);
    m = warp_max(m);
    float l = 0.0f;
    for (int c = lane; c < my_cells; c += 32) {
      const float p = m == -INFINITY ? 0.0f : expf(s_p[h][c] - m);
      s_p[h][c] = p;
      l += p;
    }
    l = warp_sum(l);
    if (lane == 0) {
      s_m[h] = m;
      s_l[h] = l;
    }
  }
  __syncthreads();
  // unnormalised P.V over this warp's cells
  float o[G][VPL];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int x = 0; x < VPL; ++x) o[h][x] = 0.0f;
#pragma unroll
  for (int j = 0; j < JMAX; ++j) {
    const int lc = j * W + warp;
    if (lc < my_cells) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float p = s_p[h][lc];
#pragma unroll
        for (int x = 0; x < VPL; ++x) o[h][x] = fmaf(p, kv_v[j][x], o[h][x]);
      }
    }
  }
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int x = 0; x < VPL; ++x) s_o[warp][h][lane * VPL + x] = o[h][x];
  __syncthreads();
  // sum over warps (fixed order) and store the partial of this split
  for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
    const int h = e / D, d = e % D;
    float acc = 0.0f;
#pragma unroll
    for (int w = 0; w < W; ++w) acc += s_o[w][h][d];
    part_o[(size_t(split) * n_q_heads + g * G + h) * D + d] = acc;
  }
  if (threadIdx.x < G) {
    const int h = threadIdx.x;
    part_ml[(size_t(split) * n_q_heads + g * G + h) * 2 + 0] = s_m[h];
    part_ml[(size_t(split) * n_q_heads + g * G + h) * 2 + 1] = s_l[h];
  }
}

// Merge the splits of one query head: out = sum_s e^(m_s-M) o_s / sum_s e^(m_s-M) l_s.
__global__ void __launch_bounds__(128) attn_combine_kernel(const float* __restrict__ part_o,
                                                           const float* __restrict__ part_ml,
                                                           float* __restrict__ out, int n_q_heads, int D,
                                                           int n_splits) {
  pdl_wait();
  const int i = blockIdx.x;
  float M = -INFINITY;
  for (int s = 0; s < n_splits; ++s) M = fmaxf(M, part_ml[(size_t(s) * n_q_heads + i) * 2]);
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float acc = 0.0f, den = 0.0f;
    if (M != -INFINITY) {
      for (int s = 0; s < n_splits; ++s) {
        const float m = part_ml[(size_t(s) * n_q_heads + i) * 2];
        if (m == -INFINITY) continue;
        const float e = expf(m - M);
        acc = fmaf(e, part_o[(size_t(s) * n_q_heads + i) * D + d], acc);
        den = fmaf(e, part_ml[(size_t(s) * n_q_heads + i) * 2 + 1], den);
      }
    }
    out[size_t(i) * D + d] = den > 0.0f ? acc / den : 0.0f;
  }
}

template <int D>
static cudaError_t launch_attn_d(const LayerView& L, const void* q, const int32_t* cells, const int32_t* n_cells,
                                 cudaStream_t s) {
  const dim3 grid(L.split.n_splits, L.cfg.n_kv_heads), block(kAttnWarps * 32);
  const int G = L.cfg.n_q_heads / L.cfg.n_kv_heads;
  const int mc = L.split.n_splits * L.split.cells_per_cta;
  const int maxc = max_cells_of(L.cfg) < mc ? max_cells_of(L.cfg) : mc;
#define QSA_ATTN_CASE(GG)                                                                                   \
  case GG:                                                                                                  \
    return launch_pdl(attn_split_kernel<D, GG>, grid, block, 0, s, 1, L.state, (const __half*)q, cells,     \
                      n_cells, (const __half*)L.k_cache, (const __half*)L.v_cache, L.part_o, L.part_ml,     \
                      L.cfg.n_kv_heads, L.split.cells_per_cta, maxc);
  switch (G) {
    QSA_ATTN_CASE(1)
    QSA_ATTN_CASE(2)
    QSA_ATTN_CASE(4)
    QSA_ATTN_CASE(8)
    default: return cudaErrorInvalidValue;
  }
#undef QSA_ATTN_CASE
}

cudaError_t launch_attend_split(const LayerView& L, const void* q, const int32_t* cells, const int32_t* n_cells,
                                float* out, cudaStream_t s) {
  cudaError_t e = L.cfg.head_dim == 128 ? launch_attn_d<128>(L, q, cells, n_cells, s)
                                        : launch_attn_d<64>(L, q, cells, n_cells, s);
  if (e != cudaSuccess) return e;
  return launch_pdl(attn_combine_kernel, dim3(L.cfg.n_q_heads), dim3(128), 0, s, 1, (const float*)L.part_o,
                    (const float*)L.part_ml, out, L.cfg.n_q_heads, L.cfg.head_dim, L.split.n_splits);
}

// ---------------------------------------------------------------------------------
// Split-KV flash decode with the split merge done in distributed shared memory.
// One cluster of CS CTAs per KV head g covers the whole cell set: CTA r stages the K
// and V rows of cells [r*Lc, (r+1)*Lc) in shared memory (16-byte cp.async, straight
// from the cache: the gather is fused), computes the f32 logits, softmax statistics and
// unnormalised P.V of the G query heads that share g, then the CTAs merge their
// (max, sum, output) partials through DSMEM and write the final output. In the
// FROM_BLOCKS form the cell ids are expanded on the fly from the selected blocks and
// the open tail (cell expansion fused in as well).
// ---------------------------------------------------------------------------------
constexpr int kAcThreads = 512;
constexpr int kAcWarps = kAcThreads / 32;

__device__ __forceinline__ void cp_async_16(void* smem_dst, const void* gsrc, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
               "l"(gsrc), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

template <int D, int G>
struct AcSmem {
  // byte offsets inside the dynamic shared memory for Lc cells per CTA
  __host__ __device__ static size_t k_off(int) { return 0; }
  __host__ __device__ static size_t v_off(int lc) { return size_t(lc) * D * 2; }
  __host__ __device__ static size_t p_off(int lc) { return size_t(lc) * D * 4; }
  __host__ __device__ static size_t o_off(int lc) { return (p_off(lc) + size_t(G) * lc * 4 + 15) / 16 * 16; }
  __host__ __device__ static size_t ml_off(int lc) { return o_off(lc) + size_t(G) * D * 4; }
  __host__ __device__ static size_t cell_off(int lc) { return ml_off(lc) + 2 * G * 4; }
  __host__ __device__ static size_t stage_off(int lc) { return (cell_off(lc) + size_t(lc) * 4 + 15) / 16 * 16; }
  __host__ __device__ static size_t bytes(int lc, int cs) { return stage_off(lc) + size_t(cs) * G * 2 * 4; }
};

template <int D, int G, int CS, bool FROM_BLOCKS>
__global__ void __launch_bounds__(kAcThreads, 1)
attn_cluster_kernel(DevState* st, const __half* __restrict__ q, const int32_t* __restrict__ ids,
                    const int32_t* __restrict__ n_ids, const __half* __restrict__ kc, const __half* __restrict__ vc,
                    float* __restrict__ out, int n_kv_heads, int cells_per_cta, int max_cells, int k_blocks) {
  using SM = AcSmem<D, G>;
  constexpr int VPL = D / 32;
  constexpr int CH = D * 2 / 16;  // 16-byte chunks per row
  extern __shared__ __align__(16) unsigned char smem[];
  const int Lc = cells_per_cta;
  __half* sK = reinterpret_cast<__half*>(smem + SM::k_off(Lc));
  __half* sV = reinterpret_cast<__half*>(smem + SM::v_off(Lc));
  float* s_p = reinterpret_cast<float*>(smem + SM::p_off(Lc));
  float* s_o = reinterpret_cast<float*>(smem + SM::o_off(Lc));
  float* s_m = reinterpret_cast<float*>(smem + SM::ml_off(Lc));
  float* s_l = s_m + G;
  int* s_cell = reinterpret_cast<int*>(smem + SM::cell_off(Lc));
  float* s_stage = reinterpret_cast<float*>(smem + SM::stage_off(Lc));  // [CS][G][2] merged (m, l)

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = int(cluster.block_rank());
  const int g = blockIdx.x / CS;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  pdl_launch_dependents();
  pdl_wait();
  const int n = ld_volatile(&st->n_ctx);
  const int n_blocks = n / kBlock;
  int total, ns = 0;
  if constexpr (FROM_BLOCKS) {
    ns = *n_ids;
    if (ns < 0 || ns > k_blocks) {
      if (blockIdx.x == 0 && tid == 0) record_status(st, QSA_ERR_BAD_INDEX);
      ns = ns < 0 ? 0 : k_blocks;
    }
    total = kBlock * ns + (n - kBlock * n_blocks);
  } else {
    total = *n_ids;
    if (total < 0 || total > max_cells) {
      if (blockIdx.x == 0 && tid == 0) record_status(st, QSA_ERR_BAD_INDEX);
      total = total < 0 ? 0 : max_cells;
    }
  }
  const int c0 = rank * Lc;
  const int cnt = max(0, min(Lc, total - c0));

  for (int i = tid; i < cnt; i += kAcThreads) {
    const int ci = c0 + i;
    int cell;
    if constexpr (FROM_BLOCKS) {
      if (ci < kBlock * ns) {
        const int b = ids[ci / kBlock];
        cell = (b >= 0 && b < n_blocks) ? kBlock * b + ci % kBlock : -1;
      } else {
        cell = kBlock * n_blocks + (ci - kBlock * ns);
      }
    } else {
      cell = ids[ci];
    }
    if (cell < 0 || cell >= n) {
      record_status(st, QSA_ERR_BAD_INDEX);
      cell = -1;
    }
    s_cell[i] = cell;
  }
  __syncthreads();
  // stage the selected K and V rows (rows of invalid cells are zero-filled)
  for (int e = tid; e < cnt * CH; e += kAcThreads) {
    const int i = e / CH, ch = e % CH;
    const int cell = s_cell[i];
    const size_t off = cell >= 0 ? ((size_t(cell) * n_kv_heads + g) * D + ch * 8) : 0;
    cp_async_16(sK + size_t(i) * D + ch * 8, kc + off, cell >= 0 ? 16 : 0);
    cp_async_16(sV + size_t(i) * D + ch * 8, vc + off, cell >= 0 ? 16 : 0);
  }
  float qv[G][VPL];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int x = 0; x < VPL; ++x) qv[h][x] = __half2float(q[(size_t(g) * G + h) * D + lane * VPL + x]);
  cp_async_commit_wait_all();
  __syncthreads();

  // logits: warp w takes cells w, w + 16, ..., four at a time so that the four
  // transposing reductions (shuffle chains) interleave
  const float scale = 1.0f / sqrtf((float)D);
  constexpr int UN = 4;
  for (int i0 = warp; i0 < cnt; i0 += kAcWarps * UN) {
    float dot[UN][G];
#pragma unroll
    for (int u = 0; u < UN; ++u) {
      const int i = i0 + u * kAcWarps;
      float kx[VPL];
      if (i < cnt) {
        if constexpr (VPL == 4) {
          const uint2 raw = *reinterpret_cast<const uint2*>(sK + size_t(i) * D + lane * 4);
          const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
          const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
          kx[0] = a.x; kx[1] = a.y; kx[2] = b.x; kx[3] = b.y;
        } else {
          const float2 a = __half22float2(*reinterpret_cast<const __half2*>(sK + size_t(i) * D + lane * 2));
          kx[0] = a.x; kx[1] = a.y;
        }
      } else {
#pragma unroll
        for (int x = 0; x < VPL; ++x) kx[x] = 0.0f;
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float a = 0.0f;
#pragma unroll
        for (int x = 0; x < VPL; ++x) a = fmaf(qv[h][x], kx[x], a);
        dot[u][h] = a;
      }
    }
    float mine[UN];
#pragma unroll
    for (int u = 0; u < UN; ++u) mine[u] = transpose_reduce<G>(dot[u], lane);
    const int h = head_of_lane<G>(lane);
#pragma unroll
    for (int u = 0; u < UN; ++u) {
      const int i = i0 + u * kAcWarps;
      if (i < cnt && (lane & (32 / G - 1)) == 0) s_p[h * Lc + i] = s_cell[i] >= 0 ? mine[u] * scale : -INFINITY;
    }
  }
  __syncthreads();
  // softmax statistics of this CTA's cells, per head
  for (int h = warp; h < G; h += kAcWarps) {
    float m = -INFINITY;
    for (int i = lane; i < cnt; i += 32) m = fmaxf(m, s_p[h * Lc + i]);
    m = warp_max(m);
    float l = 0.0f;
    for (int i = lane; i < cnt; i += 32) {
      const float p = m == -INFINITY ? 0.0f : expf(s_p[h * Lc + i] - m);
      s_p[h * Lc + i] = p;
      l += p;
    }
    l = warp_sum(l);
    if (lane == 0) {
      s_m[h] = m;
      s_l[h] = l;
    }
  }
  __syncthreads();
  // unnormalised P.V: thread -> (head, pair of dims); four independent partial sums over
  // the cells (cell i goes to partial i % 4, the cnt % 4 leftovers to partial 0), added in a fixed order
  for (int t = tid; t < G * (D / 2); t += kAcThreads) {
    const int h = t / (D / 2), d2 = t % (D / 2);
    float o0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, o1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    const float* ph = s_p + h * Lc;
    int i = 0;
    for (; i + 4 <= cnt; i += 4) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 vv = __half22float2(*reinterpret_cast<const __half2*>(sV + size_t(i + u) * D + 2 * d2));
        const float p = ph[i + u];
        o0[u] = fmaf(p, vv.x, o0[u]);
        o1[u] = fmaf(p, vv.y, o1[u]);
      }
    }
    for (; i < cnt; ++i) {  // the last cnt % 4 cells go to partial 0
      const float2 vv = __half22float2(*reinterpret_cast<const __half2*>(sV + size_t(i) * D + 2 * d2));
      const float p = ph[i];
      o0[0] = fmaf(p, vv.x, o0[0]);
      o1[0] = fmaf(p, vv.y, o1[0]);
    }
    s_o[h * D + 2 * d2] = (o0[0] + o0[1]) + (o0[2] + o0[3]);
    s_o[h * D + 2 * d2 + 1] = (o1[0] + o1[1]) + (o1[2] + o1[3]);
  }
  cluster.sync();
  // merge the CS partials: (max, sum) of every CTA first, then this CTA's output slice
  for (int t = tid; t < CS * G; t += kAcThreads) {
    const int r = t / G, h = t % G;
    const float* rm = cluster.map_shared_rank(s_m, r);
    s_stage[(r * G + h) * 2] = rm[h];
    s_stage[(r * G + h) * 2 + 1] = rm[G + h];
  }
  __syncthreads();
  constexpr int PAIRS = G * (D / 2);
  constexpr int PER = (PAIRS + CS - 1) / CS;
  for (int t = tid; t < PER; t += kAcThreads) {
    const int pidx = rank * PER + t;
    if (pidx >= PAIRS) break;
    const int h = pidx / (D / 2), d2 = pidx % (D / 2);
    float M = -INFINITY;
#pragma unroll
    for (int r = 0; r < CS; ++r) M = fmaxf(M, s_stage[(r * G + h) * 2]);
    float2 o[CS];
#pragma unroll
    for (int r = 0; r < CS; ++r) o[r] = *reinterpret_cast<const float2*>(cluster.map_shared_rank(s_o, r) + h * D + 2 * d2);
    float a0 = 0.0f, a1 = 0.0f, den = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int r = 0; r < CS; ++r) {
        const float m = s_stage[(r * G + h) * 2];
        const float e = m == -INFINITY ? 0.0f : expf(m - M);
        a0 = fmaf(e, o[r].x, a0);
        a1 = fmaf(e, o[r].y, a1);
        den = fmaf(e, s_stage[(r * G + h) * 2 + 1], den);
      }
    }
    float2 res = make_float2(0.0f, 0.0f);
    if (den > 0.0f) res = make_float2(a0 / den, a1 / den);
    *reinterpret_cast<float2*>(out + (size_t(g) * G + h) * D + 2 * d2) = res;
  }
  cluster.sync();  // keep this CTA's shared memory alive until every remote read is done
}

template <int D, int G, int CS, bool FB>
static cudaError_t set_ac_attr(size_t smem) {
  cudaError_t e = cudaFuncSetAttribute(attn_cluster_kernel<D, G, CS, FB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e == cudaSuccess && CS > 8)
    e = cudaFuncSetAttribute(attn_cluster_kernel<D, G, CS, FB>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return e;
}

template <int D, int G, int CS>
static cudaError_t launch_ac(const LayerView& L, bool from_blocks, const void* q, const int32_t* ids,
                             const int32_t* n_ids, float* out, cudaStream_t s) {
  const int lc = L.attn_cells_per_cta;
  const size_t smem = AcSmem<D, G>::bytes(lc, CS);
  const dim3 grid(L.cfg.n_kv_heads * CS), block(kAcThreads);
  const int mc = max_cells_of(L.cfg), kb = L.cfg.top_k_tokens / kBlock;
  if (from_blocks)
    return launch_pdl(attn_cluster_kernel<D, G, CS, true>, grid, block, smem, s, CS, L.state, (const __half*)q, ids,
                      n_ids, (const __half*)L.k_cache, (const __half*)L.v_cache, out, L.cfg.n_kv_heads, lc, mc, kb);
  return launch_pdl(attn_cluster_kernel<D, G, CS, false>, grid, block, smem, s, CS, L.state, (const __half*)q, ids,
                    n_ids, (const __half*)L.k_cache, (const __half*)L.v_cache, out, L.cfg.n_kv_heads, lc, mc, kb);
}

template <int D, int G>
static cudaError_t launch_ac_g(const LayerView& L, bool fb, const void* q, const int32_t* ids, const int32_t* n_ids,
                               float* out, cudaStream_t s) {
  return L.attn_cluster == 16 ? launch_ac<D, G, 16>(L, fb, q, ids, n_ids, out, s)
                              : launch_ac<D, G, 8>(L, fb, q, ids, n_ids, out, s);
}

template <int D>
static cudaError_t launch_ac_d(const LayerView& L, bool fb, const void* q, const int32_t* ids, const int32_t* n_ids,
                               float* out, cudaStream_t s) {
  switch (L.cfg.n_q_heads / L.cfg.n_kv_heads) {
    case 1: return launch_ac_g<D, 1>(L, fb, q, ids, n_ids, out, s);
    case 2: return launch_ac_g<D, 2>(L, fb, q, ids, n_ids, out, s);
    case 4: return launch_ac_g<D, 4>(L, fb, q, ids, n_ids, out, s);
    case 8: return launch_ac_g<D, 8>(L, fb, q, ids, n_ids, out, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_attend(const LayerView& L, const void* q, const int32_t* cells, const int32_t* n_cells, float* out,
                          cudaStream_t s) {
  return L.cfg.head_dim == 128 ? launch_ac_d<128>(L, false, q, cells, n_cells, out, s)
                               : launch_ac_d<64>(L, false, q, cells, n_cells, out, s);
}

cudaError_t launch_attend_selected(const LayerView& L, const void* q, const int32_t* sel, const int32_t* n_sel,
                                   float* out, cudaStream_t s) {
  return L.cfg.head_dim == 128 ? launch_ac_d<128>(L, true, q, sel, n_sel, out, s)
                               : launch_ac_d<64>(L, true, q, sel, n_sel, out, s);
}

// Cluster size and cells per CTA for a configuration, plus the kernel attributes they
// need; called once per context, outside any stream capture.
template <int D, int G>
static cudaError_t plan_ac_g(const qsa_config& c, int* cluster, int* lc) {
  const int mc = max_cells_of(c);
  for (int cs : {16, 8}) {
    const int l = (mc + cs - 1) / cs;
    const size_t smem = AcSmem<D, G>::bytes(l, cs);
    if (smem > 220 * 1024) continue;
    cudaError_t e = cs == 16 ? set_ac_attr<D, G, 16, false>(smem) : set_ac_attr<D, G, 8, false>(smem);
    if (e == cudaSuccess) e = cs == 16 ? set_ac_attr<D, G, 16, true>(smem) : set_ac_attr<D, G, 8, true>(smem);
    if (e != cudaSuccess) {
      cudaGetLastError();
      continue;
    }
    // every KV head's cluster must be able to run at the same time
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(c.n_kv_heads * cs);
    cfg.blockDim = dim3(kAcThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = cs;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int active = 0;
    e = cs == 16 ? cudaOccupancyMaxActiveClusters(&active, attn_cluster_kernel<D, G, 16, true>, &cfg)
                 : cudaOccupancyMaxActiveClusters(&active, attn_cluster_kernel<D, G, 8, true>, &cfg);
    if (e != cudaSuccess) {
      cudaGetLastError();
      continue;
    }
    if (active >= (cs == 16 ? c.n_kv_heads : 1)) {
      *cluster = cs;
      *lc = l;
      return cudaSuccess;
    }
  }
  return cudaErrorNotSupported;
}

cudaError_t plan_attention(const qsa_config& c, int* cluster, int* cells_per_cta) {
  const int G = c.n_q_heads / c.n_kv_heads;
  if (c.head_dim == 128) {
    switch (G) {
      case 1: return plan_ac_g<128, 1>(c, cluster, cells_per_cta);
      case 2: return plan_ac_g<128, 2>(c, cluster, cells_per_cta);
      case 4: return plan_ac_g<128, 4>(c, cluster, cells_per_cta);
      case 8: return plan_ac_g<128, 8>(c, cluster, cells_per_cta);
    }
  } else {
    switch (G) {
      case 1: return plan_ac_g<64, 1>(c, cluster, cells_per_cta);
      case 2: return plan_ac_g<64, 2>(c, cluster, cells_per_cta);
      case 4: return plan_ac_g<64, 4>(c, cluster, cells_per_cta);
      case 8: return plan_ac_g<64, 8>(c, cluster, cells_per_cta);
    }
  }
  return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------------------------
// Attention for callers that cannot allocate device memory (qsa_sparse_attend_noalloc).
// The split-KV partials and the small state block that the attention kernels use as
// scratch live in one fixed array compiled into the library, so the caller passes only
// its inputs and its output. Every GPU that loads the library holds this array until
// the process exits, and all calls on a device share it.
// ---------------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[QSA_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices];  // device address of g_noalloc_scratch, per device
int g_noalloc_sms[kMaxDevices];

// Once per device, with that device current: look up the array's device address (host
// code cannot use the symbol itself, which is only a host-side stand-in).
cudaError_t noalloc_setup(void** addr, int* n_sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_sms[dev] = sms;
    g_noalloc_addr[dev] = p;
  }
  *addr = g_noalloc_addr[dev];
  *n_sms = g_noalloc_sms[dev];
  return cudaSuccess;
}

bool aligned_to(const void* p, uintptr_t a) { return p && (reinterpret_cast<uintptr_t>(p) % a) == 0; }
}  // namespace

}  // namespace qsa

extern "C" qsa_status qsa_sparse_attend_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                                int32_t n_ctx, const int32_t* cells, const int32_t* n_cells,
                                                float* out, int32_t n_q_heads, int32_t n_kv_heads,
                                                int32_t head_dim, int32_t top_k_tokens, qsa_stream_t stream) {
  using namespace qsa;
  if (!aligned_to(q, 16) || !aligned_to(k_cache, 16) || !aligned_to(v_cache, 16) || !aligned_to(cells, 16) ||
      !aligned_to(n_cells, 4) || !aligned_to(out, 16) || n_ctx < 0)
    return QSA_ERR_INVALID_ARG;
  if ((head_dim != 64 && head_dim != 128) || n_kv_heads < 1 || n_q_heads < 1 || n_q_heads % n_kv_heads ||
      top_k_tokens < kBlock || top_k_tokens % kBlock)
    return QSA_ERR_UNSUPPORTED;
  const int g = n_q_heads / n_kv_heads;
  if (g != 1 && g != 2 && g != 4 && g != 8) return QSA_ERR_UNSUPPORTED;
  void* base = nullptr;
  int n_sms = 0;
  if (noalloc_setup(&base, &n_sms) != cudaSuccess) return QSA_ERR_CUDA;

  LayerView v{};
  v.cfg.n_layers = 1;
  v.cfg.max_ctx = n_ctx;
  v.cfg.top_k_tokens = top_k_tokens;
  v.cfg.n_q_heads = n_q_heads;
  v.cfg.n_kv_heads = n_kv_heads;
  v.cfg.head_dim = head_dim;
  v.k_cache = const_cast<void*>(k_cache);
  v.v_cache = const_cast<void*>(v_cache);
  v.split = attn_split(v.cfg, n_sms);
  v.n_sms = n_sms;
  // scratch layout: state block | (max, sum) pairs | partial outputs
  const size_t ml_bytes = align256(size_t(v.split.n_splits) * n_q_heads * 2 * sizeof(float));
  const size_t o_bytes = size_t(v.split.n_splits) * n_q_heads * head_dim * sizeof(float);
  if (sizeof(DevState) + ml_bytes + o_bytes > QSA_NOALLOC_SCRATCH_BYTES) return QSA_ERR_CAPACITY;
  char* p = static_cast<char*>(base);
  v.state = reinterpret_cast<DevState*>(p);
  v.part_ml = reinterpret_cast<float*>(p + sizeof(DevState));
  v.part_o = reinterpret_cast<float*>(p + sizeof(DevState) + ml_bytes);
  // the state block keeps the previous call's contents: set n_ctx and clear the status
  if (launch_set_state(v, n_ctx, 0, kSetRestore, (cudaStream_t)stream) != cudaSuccess) return QSA_ERR_CUDA;
  if (launch_attend_split(v, q, cells, n_cells, out, (cudaStream_t)stream) != cudaSuccess) return QSA_ERR_CUDA;
  return QSA_OK;
}
