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
#include <cuda_fp8.h>

#include <cooperative_groups.h>

#include <mutex>

#include "qsa_device.cuh"
#include "qsa_sm100.cuh"
#include "qsa_timeline.cuh"

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
// unnormalised P.V of the G query heads that share g, then pushes its (max, sum, output)
// partials through DSMEM to the CTAs that own each output slice, which merge them after
// a single cluster barrier and write the final output. In the
// FROM_BLOCKS form the cell ids are expanded on the fly from the selected blocks and
// the open tail (cell expansion fused in as well). With gridDim.y = T > 1 (multi-query
// step), the clusters of row u serve the query of token n_ctx - T + u: its q, id and
// output rows, and only the first n_ctx - T + u + 1 tokens (its own open tail).
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

// Warp-level tensor-core helpers (f16 inputs, f32 accumulation). The contractions here
// are tiny (8 query heads x ~129 cells per CTA), below the 64/128-row tiles of tcgen05,
// so the warp-synchronous m16n8k16 form is used; it keeps the logits and P.V off the
// CUDA cores, whose issue rate bounded this kernel. Both products are taken transposed
// (cells, resp. output dims, as the 16 MMA rows and the query heads as the 8 columns),
// so that no MMA row is padding.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))));
}
__device__ __forceinline__ void ldsm_x2(uint32_t (&r)[2], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))));
}

// Shared memory of attn_cluster_kernel for Lc cells per CTA (LP = Lc rounded up to 16).
// K and V rows are padded to D + 8 halves and P rows to LP + 8 halves so that the 8 row
// addresses of every ldmatrix fall in distinct 16-byte bank groups.
template <int D, int G>
struct AcSmem {
  static constexpr int RS = D + 8;  // K/V row stride (halves)
  __host__ __device__ static int lp(int lc) { return (lc + 15) & ~15; }
  __host__ __device__ static int ps(int lc) { return lp(lc) + 8; }  // P row stride (halves)
  __host__ __device__ static size_t k_off(int) { return 0; }
  __host__ __device__ static size_t v_off(int lc) { return size_t(lp(lc)) * RS * 2; }
  __host__ __device__ static size_t p_off(int lc) { return 2 * v_off(lc); }
  __host__ __device__ static size_t o_off(int lc) { return p_off(lc) + size_t(8) * ps(lc) * 2; }
  __host__ __device__ static size_t red_off(int lc) { return o_off(lc) + size_t(G) * D * 4; }     // 2 x 16 x 8 f32
  __host__ __device__ static size_t ml_off(int lc) { return red_off(lc) + 2 * 16 * 8 * 4; }        // 2G f32
  __host__ __device__ static size_t cell_off(int lc) { return ml_off(lc) + 16 * 4; }
  __host__ __device__ static size_t stage_off(int lc) { return (cell_off(lc) + size_t(lp(lc)) * 4 + 15) / 16 * 16; }
  // output pairs (2 dims of one head) each CTA of a cluster of cs merges
  __host__ __device__ static int per(int cs) { return (G * (D / 2) + cs - 1) / cs; }
  // inbox of this CTA's output slice: [cs source CTAs][per] float2
  __host__ __device__ static size_t in_off(int lc, int cs) { return (stage_off(lc) + size_t(cs) * G * 2 * 4 + 15) / 16 * 16; }
  // the query rows of this KV head (8 rows, heads >= G zero), staged with the K/V rows
  __host__ __device__ static size_t q_off(int lc, int cs) { return in_off(lc, cs) + size_t(cs) * per(cs) * 8; }
  __host__ __device__ static size_t bytes(int lc, int cs) { return q_off(lc, cs) + size_t(8) * RS * 2; }
};

// FP8 (K/V cache in e4m3 with a per-row scale): each staged row is converted to f16 as
// code * scale (one rounding) on its way into shared memory; everything after the
// staging is the f16 path.
__device__ __forceinline__ uint4 fp8x16_to_half(uint4 codes, float scale, int half_index) {
  // codes holds 16 e4m3 bytes; returns the 8 halves of bytes [8*half_index, 8*half_index+8)
  const uint32_t w0 = half_index ? codes.z : codes.x, w1 = half_index ? codes.w : codes.y;
  uint32_t r[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t w = j < 2 ? w0 : w1;
    const __nv_fp8x2_storage_t pair = (__nv_fp8x2_storage_t)((w >> (16 * (j & 1))) & 0xffffu);
    const float2 f = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3)));
    const __half2 h = __floats2half2_rn(f.x * scale, f.y * scale);
    r[j] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return make_uint4(r[0], r[1], r[2], r[3]);
}

// The register cap keeps a CTA (512 threads) small enough to share an SM with a CTA of
// the next layer's scan, which launches while this kernel runs.
template <int D, int G, int CS, bool FROM_BLOCKS, bool FP8>
__global__ void __maxnreg__(80)
attn_cluster_kernel(DevState* st, const __half* __restrict__ q, const int32_t* __restrict__ ids,
                    const int32_t* __restrict__ n_ids, const void* __restrict__ kc_raw,
                    const void* __restrict__ vc_raw, float* __restrict__ out, int n_kv_heads, int cells_per_cta,
                    int max_cells, int k_blocks, const float* __restrict__ kv_scales, float* __restrict__ lse_out,
                    int warm) {
  const __half* __restrict__ kc = static_cast<const __half*>(kc_raw);
  const __half* __restrict__ vc = static_cast<const __half*>(vc_raw);
  using SM = AcSmem<D, G>;
  constexpr int RS = SM::RS;
  constexpr int KSTEPS = D / 16;
  constexpr int CH = D * 2 / 16;  // 16-byte chunks per row
  static_assert(G <= 8, "the 8 MMA columns hold the query heads of one KV head");
  extern __shared__ __align__(16) unsigned char smem[];
  const int Lc = cells_per_cta;
  const int LP = SM::lp(Lc), PS = SM::ps(Lc);
  __half* sK = reinterpret_cast<__half*>(smem + SM::k_off(Lc));
  __half* sV = reinterpret_cast<__half*>(smem + SM::v_off(Lc));
  __half* sP = reinterpret_cast<__half*>(smem + SM::p_off(Lc));
  float* s_o = reinterpret_cast<float*>(smem + SM::o_off(Lc));
  float* s_rmax = reinterpret_cast<float*>(smem + SM::red_off(Lc));   // [16 warps][8 query heads]
  float* s_rsum = s_rmax + 16 * 8;
  float* s_m = reinterpret_cast<float*>(smem + SM::ml_off(Lc));       // [G], then s_l [G]
  float* s_l = s_m + G;
  int* s_cell = reinterpret_cast<int*>(smem + SM::cell_off(Lc));
  __half* sQ = reinterpret_cast<__half*>(smem + SM::q_off(Lc, CS));
  float* s_stage = reinterpret_cast<float*>(smem + SM::stage_off(Lc));  // [CS][G][2] merged (m, l)

  __shared__ uint64_t s_merge_bar;  // this CTA's slice: every CTA's partial has landed
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = int(cluster.block_rank());
  const int g = blockIdx.x / CS;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // m16n8k16 fragment coordinates: group gq (row gq and gq + 8 of A and D, column gq of B)
  // and thread tq in the group (columns 2tq, 2tq + 1 of D)
  const int gq = lane >> 2, tq = lane & 3;
  const int u = blockIdx.y, n_back = gridDim.y - 1 - blockIdx.y;
  q += size_t(u) * n_kv_heads * G * D;
  out += size_t(u) * n_kv_heads * G * D;
  if (lse_out) lse_out += size_t(u) * n_kv_heads * G;
  ids += size_t(u) * (FROM_BLOCKS ? k_blocks : max_cells);
  n_ids += u;

  if (tid == 0) {  // one arrival per source CTA, plus the bytes each announces
    sm100::mbar_init(&s_merge_bar, CS);
    sm100::fence_mbar_init();
  }
  if (tid == 0) QSA_TL(st, kTlAttn, kTlEntry);
  cluster_arrive_relaxed();  // paired with cluster_wait() before the partials are pushed
  // With `warm` (the decode step, where this kernel launches while the selection still
  // runs): two passes over the same code. Pass 0 runs before the dependency wait with no
  // cells (zero rows, nothing read from global memory, only this CTA's shared memory
  // written), so that the instructions of the staging, logits and P.V phases are in the
  // SM's instruction cache when pass 1 runs them on the selected cells. The pass number
  // goes through a register move the compiler cannot see into, so that it keeps one copy
  // of the loop body instead of peeling the first pass.
#ifdef QSA_TIMELINE
  long long cyc0 = 0;  // clock64 deltas from the cells known, min..max over the CTAs
#define QSA_ACYC(pt) if (tid == 0) QSA_TL_VALUE(st, kTlAttnCyc, pt, uint32_t(clock64() - cyc0))
#else
#define QSA_ACYC(pt) ((void)0)
#endif
#pragma unroll 1
  for (int pass_i = warm ? 0 : 1; pass_i < 2; ++pass_i) {
    int pass;
    asm volatile("mov.b32 %0, %1;" : "=r"(pass) : "r"(pass_i));
    const int c0 = rank * Lc;
    int n = 0, n_blocks = 0, ns = 0, id_spec = 0, cnt = 0;
    if (pass) {
      pdl_wait();
      // the next kernel (in the decode step, the next layer's scan, whose prologue and L2
      // prefetch of the pooled keys are heavy) launches now, beside this kernel's own
      // loads and math, rather than while the selection before it runs
      pdl_launch_dependents();
      if (tid == 0) QSA_TL(st, kTlAttn, kTlWait);
      const int n_full = ld_volatile(&st->n_ctx);
      // this thread's id, loaded in the same round trip as the counts (clamped into the
      // id buffer, checked against the counts below)
      if (tid < Lc) {
        const int ci = c0 + tid;
        id_spec = FROM_BLOCKS ? ids[min(ci / kBlock, k_blocks - 1)] : ids[min(ci, max_cells - 1)];
      }
      const int n_ids_v = *n_ids;
      asm volatile("" ::"r"(id_spec), "r"(n_ids_v), "r"(n_full));  // keep the loads ahead of the branches
      n = n_full - n_back;  // tokens this query sees
      if (n < 0) {
        if (rank == 0 && tid == 0) record_status(st, QSA_ERR_STATE);
        n = 0;
      }
      n_blocks = n / kBlock;
      int total;
      if constexpr (FROM_BLOCKS) {
        ns = n_ids_v;
        if (ns < 0 || ns > k_blocks) {
          if (blockIdx.x == 0 && tid == 0) record_status(st, QSA_ERR_BAD_INDEX);
          ns = ns < 0 ? 0 : k_blocks;
        }
        total = kBlock * ns + (n - kBlock * n_blocks);
      } else {
        total = n_ids_v;
        if (total < 0 || total > max_cells) {
          if (blockIdx.x == 0 && tid == 0) record_status(st, QSA_ERR_BAD_INDEX);
          total = total < 0 ? 0 : max_cells;
        }
      }
      cnt = max(0, min(Lc, total - c0));
    }

    for (int i = tid; i < LP; i += kAcThreads) {
      int cell = -1;
      if (i < cnt) {
        const int ci = c0 + i;
        if constexpr (FROM_BLOCKS) {
          if (ci < kBlock * ns) {
            const int b = i == tid ? id_spec : ids[ci / kBlock];
            cell = (b >= 0 && b < n_blocks) ? kBlock * b + ci % kBlock : -1;
          } else {
            cell = kBlock * n_blocks + (ci - kBlock * ns);
          }
        } else {
          cell = i == tid ? id_spec : ids[ci];
        }
        if (cell < 0 || cell >= n) {
          record_status(st, QSA_ERR_BAD_INDEX);
          cell = -1;
        }
      }
      s_cell[i] = cell;
    }
    __syncthreads();
    if (pass && tid == 0) QSA_TL(st, kTlAttn2, 0);  // cells known
#ifdef QSA_TIMELINE
    cyc0 = clock64();
#endif
    // stage the selected K and V rows (rows of invalid or padding cells are zero-filled)
    if constexpr (!FP8) {
      for (int e = tid; e < LP * CH; e += kAcThreads) {
        const int i = e / CH, ch = e % CH;
        const int cell = s_cell[i];
        const size_t off = cell >= 0 ? ((size_t(cell) * n_kv_heads + g) * D + ch * 8) : 0;
        cp_async_16(sK + size_t(i) * RS + ch * 8, kc + off, cell >= 0 ? 16 : 0);
        cp_async_16(sV + size_t(i) * RS + ch * 8, vc + off, cell >= 0 ? 16 : 0);
      }
    } else {
      // 16 e4m3 codes per 16-byte load; a row is D/16 of them
      constexpr int CH8 = D / 16;
      const unsigned char* kc8 = static_cast<const unsigned char*>(kc_raw);
      const unsigned char* vc8 = static_cast<const unsigned char*>(vc_raw);
#pragma unroll 2
      for (int e = tid; e < LP * CH8; e += kAcThreads) {
        const int i = e / CH8, ch = e % CH8;
        const int cell = s_cell[i];
        uint4 kq = make_uint4(0u, 0u, 0u, 0u), vq = kq;
        float2 sc = make_float2(0.0f, 0.0f);
        if (cell >= 0) {
          const size_t row = size_t(cell) * n_kv_heads + g;
          kq = *reinterpret_cast<const uint4*>(kc8 + row * D + ch * 16);
          vq = *reinterpret_cast<const uint4*>(vc8 + row * D + ch * 16);
          sc = *reinterpret_cast<const float2*>(kv_scales + row * 2);
        }
        __half* kd = sK + size_t(i) * RS + ch * 16;
        __half* vd = sV + size_t(i) * RS + ch * 16;
        *reinterpret_cast<uint4*>(kd) = fp8x16_to_half(kq, sc.x, 0);
        *reinterpret_cast<uint4*>(kd + 8) = fp8x16_to_half(kq, sc.x, 1);
        *reinterpret_cast<uint4*>(vd) = fp8x16_to_half(vq, sc.y, 0);
        *reinterpret_cast<uint4*>(vd + 8) = fp8x16_to_half(vq, sc.y, 1);
      }
    }
    // the query rows of KV head g in the same copy group (rows >= G zero-filled), so that
    // they arrive with the K/V rows instead of after them
    for (int e = tid; e < 8 * CH; e += kAcThreads) {
      const int h = e / CH, ch = e % CH;
      const bool ok = pass && h < G;
      cp_async_16(sQ + h * RS + ch * 8, q + (ok ? (size_t(g) * G + h) * D + ch * 8 : 0), ok ? 16 : 0);
    }
    cp_async_commit_wait_all();
    __syncthreads();
    if (pass && tid == 0) QSA_TL(st, kTlAttn, kTlA);  // rows staged
    if (pass) QSA_ACYC(0);

    // ---- logits^T = K q^T: warp w takes cells [16w, 16w+16) as the 16 MMA rows, the
    //      query heads are the 8 columns, so no MMA row is padding. Lane (gq, tq) holds
    //      cells 16w+gq and 16w+gq+8 for heads 2tq and 2tq+1. ----
    const float scale = 1.0f / sqrtf((float)D);
    const int MT = LP / 16;  // <= 16 cell tiles
    float lg[2][2];          // [cell gq, gq + 8][head 2tq, 2tq + 1]
    float rmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int r = 0; r < 2; ++r) lg[r][0] = lg[r][1] = -INFINITY;
    if (warp < MT) {  // warp-uniform
      // B fragments (column n = query head n): two k-steps per ldmatrix.x4 of the query rows
      uint32_t qb[KSTEPS][2];
      const __half* qrow = sQ + size_t(lane & 7) * RS + (lane >> 3) * 8;
#pragma unroll
      for (int ks = 0; ks < KSTEPS; ks += 2) {
        uint32_t t[4];
        ldsm_x4(t, qrow + ks * 16);  // heads 0..7, dims ks*16 + {0..7, 8..15, 16..23, 24..31}
        qb[ks][0] = t[0];
        qb[ks][1] = t[1];
        qb[ks + 1][0] = t[2];
        qb[ks + 1][1] = t[3];
      }
      // two accumulators (even and odd k-steps) halve the dependent MMA chain
      float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f}, acc1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      const __half* ka = sK + size_t(warp * 16 + (lane & 15)) * RS + (lane >> 4) * 8;
#pragma unroll
      for (int ks = 0; ks < KSTEPS; ks += 2) {
        uint32_t a[4], a1[4];
        ldsm_x4(a, ka + ks * 16);  // cells 16w + {0..7, 8..15}, dims ks*16 + {0..7, 8..15}
        ldsm_x4(a1, ka + ks * 16 + 16);
        mma_16816(acc, a[0], a[1], a[2], a[3], qb[ks][0], qb[ks][1]);
        mma_16816(acc1, a1[0], a1[1], a1[2], a1[3], qb[ks + 1][0], qb[ks + 1][1]);
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[c] += acc1[c];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int i = warp * 16 + gq + 8 * r;
        const bool valid = i < cnt && s_cell[i] >= 0;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          lg[r][c] = (valid && 2 * tq + c < G) ? acc[2 * r + c] * scale : -INFINITY;
          rmax[c] = fmaxf(rmax[c], lg[r][c]);
        }
      }
    }
#pragma unroll
    for (int c = 0; c < 2; ++c) {
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) rmax[c] = fmaxf(rmax[c], __shfl_xor_sync(0xffffffffu, rmax[c], off));
    }
    if (gq == 0) *reinterpret_cast<float2*>(s_rmax + warp * 8 + 2 * tq) = make_float2(rmax[0], rmax[1]);
    __syncthreads();
    if (pass && tid == 0) QSA_TL(st, kTlAttn2, 1);  // logits done
    if (pass) QSA_ACYC(1);
    float m[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int w = 0; w < 16; ++w) {
      const float2 mw = *reinterpret_cast<const float2*>(s_rmax + w * 8 + 2 * tq);
      m[0] = fmaxf(m[0], mw.x);
      m[1] = fmaxf(m[1], mw.y);
    }
    // probabilities, rounded to f16 for the P.V product (P stored head-major, [head][cell]);
    // the row sums use the rounded values
    float psum[2] = {0.0f, 0.0f};
    if (warp < MT) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float p = 0.0f;  // exp(d) as 2^(d log2 e) on the MUFU unit (relative error ~2^-22)
          if (m[c] != -INFINITY) {
            const float x = (lg[r][c] - m[c]) * 1.4426950408889634f;
            asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(p) : "f"(x));
          }
          const __half h = __float2half_rn(p);
          sP[size_t(2 * tq + c) * PS + warp * 16 + gq + 8 * r] = h;
          psum[c] += __half2float(h);
        }
      }
    }
#pragma unroll
    for (int c = 0; c < 2; ++c) {
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) psum[c] += __shfl_xor_sync(0xffffffffu, psum[c], off);
    }
    if (gq == 0) *reinterpret_cast<float2*>(s_rsum + warp * 8 + 2 * tq) = make_float2(psum[0], psum[1]);
    __syncthreads();
    if (warp == D / 16 && lane < G) {  // the heads' max and sum, on a warp without P.V work
      float mm = -INFINITY, ll = 0.0f;
#pragma unroll
      for (int w = 0; w < 16; ++w) {
        mm = fmaxf(mm, s_rmax[w * 8 + lane]);
        ll += s_rsum[w * 8 + lane];
      }
      s_m[lane] = mm;
      s_l[lane] = ll;
    }
    // ---- unnormalised O^T = V^T P^T: warp w takes output dims [16w, 16w+16) as the 16
    //      MMA rows (V^T tiles by transposing loads of the cell-major rows), the heads are
    //      the 8 columns; all cells in 16-cell steps ----
    if (warp < D / 16) {
      float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f}, acc1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      const __half* va = sV + size_t((lane & 7) + ((lane >> 4) & 1) * 8) * RS + warp * 16 + ((lane >> 3) & 1) * 8;
      const __half* pb = sP + size_t(lane & 7) * PS + (lane >> 3) * 8;
      int kc16 = 0;
      for (; kc16 + 1 < MT; kc16 += 2) {  // two accumulators (even and odd cell tiles)
        uint32_t a[4], a1[4], b[4];
        ldsm_x4_trans(a, va + size_t(kc16) * 16 * RS);  // V cells kc16*16 + {0..7, 8..15}, dims 16w + {0..7, 8..15}
        ldsm_x4_trans(a1, va + size_t(kc16 + 1) * 16 * RS);
        ldsm_x4(b, pb + kc16 * 16);                       // P heads 0..7, cells kc16*16 + {0..7, ..., 24..31}
        mma_16816(acc, a[0], a[1], a[2], a[3], b[0], b[1]);
        mma_16816(acc1, a1[0], a1[1], a1[2], a1[3], b[2], b[3]);
      }
      if (kc16 < MT) {
        uint32_t a[4], b[2];
        ldsm_x4_trans(a, va + size_t(kc16) * 16 * RS);
        ldsm_x2(b, pb + kc16 * 16);
        mma_16816(acc, a[0], a[1], a[2], a[3], b[0], b[1]);
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[c] += acc1[c];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
#pragma unroll
        for (int c = 0; c < 2; ++c)
          if (2 * tq + c < G) s_o[(2 * tq + c) * D + warp * 16 + gq + 8 * r] = acc[2 * r + c];
      }
    }
    __syncthreads();  // s_o, s_m and s_l are complete (and pass 0's readers are done)
    if (pass && tid == 0) QSA_TL(st, kTlAttn2, 2);  // P.V done
    if (pass) QSA_ACYC(2);
  }
  // ---- merge: CTA r owns output pairs [r*PER, (r+1)*PER) (2 dims of one head each).
  //      Every CTA sends its (max, sum) per head and its partial of each slice into the
  //      owner's shared memory with st.async, whose bytes count on the owner's mbarrier,
  //      and announces them with one arrival there; each owner waits on its own mbarrier
  //      (no cluster-wide barrier on the way) and merges its slice from local memory. A
  //      relaxed cluster barrier, arrived once a CTA holds all its data, keeps every CTA
  //      alive until then. ----
  constexpr int PAIRS = G * (D / 2);
  constexpr int PER = (PAIRS + CS - 1) / CS;
  float2* s_in = reinterpret_cast<float2*>(smem + SM::in_off(Lc, CS));  // [CS][PER]
  cluster_wait();   // every CTA of the cluster has started: its shared memory may be written
  if (tid == 0) QSA_TL(st, kTlAttn2, 3);
  for (int pidx = tid; pidx < PAIRS; pidx += kAcThreads) {
    const int h = pidx / (D / 2), d2 = pidx % (D / 2), owner = pidx / PER;
    const float2 v = *reinterpret_cast<const float2*>(s_o + h * D + 2 * d2);
    sm100::st_async_v2(sm100::cluster_addr(s_in + rank * PER + pidx % PER, owner), __float_as_uint(v.x),
                       __float_as_uint(v.y), sm100::cluster_addr(&s_merge_bar, owner));
  }
  for (int t = tid; t < CS * G; t += kAcThreads) {
    const int owner = t / G, h = t % G;
    sm100::st_async_v2(sm100::cluster_addr(s_stage + (rank * G + h) * 2, owner), __float_as_uint(s_m[h]),
                       __float_as_uint(s_l[h]), sm100::cluster_addr(&s_merge_bar, owner));
  }
  // every source sends each owner PER output pairs and G (max, sum) pairs
  if (tid < CS) sm100::mbar_arrive_expect_tx_remote(sm100::cluster_addr(&s_merge_bar, tid), uint32_t(PER + G) * 8u);
  if (tid == 0) QSA_TL(st, kTlAttn2, 4);  // pushed
  if (!sm100::mbar_wait_cluster(&s_merge_bar, 0)) {
    if (tid == 0) record_status(st, QSA_ERR_TIMEOUT);
    (void)sm100::mbar_wait_cluster(&s_merge_bar, 0);  // stores still in flight land before this CTA leaves
  }
  cluster_arrive_relaxed();  // this CTA's data is all here; paired with the wait before exit
  if (tid == 0) QSA_TL(st, kTlAttn, kTlB);
  QSA_ACYC(3);
  // CS lanes per output pair, lane r merging source CTA r's partial; shuffles within the
  // aligned CS-lane group combine them (max, then the weighted sums)
  static_assert(PAIRS % CS == 0 && (PER * CS) % 32 == 0 && 32 % CS == 0, "whole warps, aligned lane groups");
  for (int i = tid; i < PER * CS; i += kAcThreads) {
    const int t = i / CS, r = i % CS;
    const int pidx = rank * PER + t;
    const int h = pidx / (D / 2), d2 = pidx % (D / 2);
    const float mr = s_stage[(r * G + h) * 2];
    float M = mr;
#pragma unroll
    for (int off = CS / 2; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float e = (M == -INFINITY || mr == -INFINITY) ? 0.0f : expf(mr - M);
    const float2 o = s_in[r * PER + t];
    float a0 = e * o.x, a1 = e * o.y, den = e * s_stage[(r * G + h) * 2 + 1];
#pragma unroll
    for (int off = CS / 2; off >= 1; off >>= 1) {
      a0 += __shfl_xor_sync(0xffffffffu, a0, off);
      a1 += __shfl_xor_sync(0xffffffffu, a1, off);
      den += __shfl_xor_sync(0xffffffffu, den, off);
    }
    if (r == 0) {
      float2 res = make_float2(0.0f, 0.0f);
      if (den > 0.0f) res = make_float2(a0 / den, a1 / den);
      *reinterpret_cast<float2*>(out + (size_t(g) * G + h) * D + 2 * d2) = res;
      // log-sum-exp of the head's scaled logits over all its cells (a context-parallel
      // shard's partial): max + log(sum of exp(logit - max)); -inf with no cells
      if (lse_out && d2 == 0) lse_out[size_t(g) * G + h] = den > 0.0f ? M + logf(den) : -INFINITY;
    }
  }
  cluster_wait();  // every CTA holds its data: nothing is still arriving anywhere
  if (tid == 0) QSA_TL(st, kTlAttn, kTlExit);
  QSA_ACYC(4);
#undef QSA_ACYC
}

template <int D, int G, int CS, bool FB, bool FP8>
static cudaError_t set_ac_attr1(size_t smem) {
  cudaError_t e = cudaFuncSetAttribute(attn_cluster_kernel<D, G, CS, FB, FP8>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attn_cluster_kernel<D, G, CS, FB, FP8>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             kCarveoutMaxShared);
  if (e == cudaSuccess && CS > 8)
    e = cudaFuncSetAttribute(attn_cluster_kernel<D, G, CS, FB, FP8>, cudaFuncAttributeNonPortableClusterSizeAllowed,
                             1);
  return e;
}

template <int D, int G, int CS, bool FB>
static cudaError_t set_ac_attr(size_t smem) {
  cudaError_t e = set_ac_attr1<D, G, CS, FB, false>(smem);
  return e == cudaSuccess ? set_ac_attr1<D, G, CS, FB, true>(smem) : e;
}

template <int D, int G, int CS>
static cudaError_t launch_ac(const LayerView& L, bool from_blocks, const void* q, const int32_t* ids,
                             const int32_t* n_ids, float* out, cudaStream_t s, int n_queries, float* lse, int warm) {
  const int lc = L.attn_cells_per_cta;
  const size_t smem = AcSmem<D, G>::bytes(lc, CS);
  const dim3 grid(L.cfg.n_kv_heads * CS, n_queries), block(kAcThreads);
  const int mc = max_cells_of(L.cfg), kb = L.cfg.top_k_tokens / kBlock;
  const bool fp8 = L.cfg.kv_format == QSA_KV_FP8;
  const float* scl = L.kv_scales;
#define QSA_AC_LAUNCH(FB, F8)                                                                                    \
  launch_pdl(attn_cluster_kernel<D, G, CS, FB, F8>, grid, block, smem, s, CS, L.state, (const __half*)q, ids, n_ids, \
             (const void*)L.k_cache, (const void*)L.v_cache, out, L.cfg.n_kv_heads, lc, mc, kb, scl, lse, warm)
  if (from_blocks) return fp8 ? QSA_AC_LAUNCH(true, true) : QSA_AC_LAUNCH(true, false);
  return fp8 ? QSA_AC_LAUNCH(false, true) : QSA_AC_LAUNCH(false, false);
#undef QSA_AC_LAUNCH
}

template <int D, int G>
static cudaError_t launch_ac_g(const LayerView& L, bool fb, const void* q, const int32_t* ids, const int32_t* n_ids,
                               float* out, cudaStream_t s, int nq, float* lse, int warm) {
  return L.attn_cluster == 16 ? launch_ac<D, G, 16>(L, fb, q, ids, n_ids, out, s, nq, lse, warm)
                              : launch_ac<D, G, 8>(L, fb, q, ids, n_ids, out, s, nq, lse, warm);
}

template <int D>
static cudaError_t launch_ac_d(const LayerView& L, bool fb, const void* q, const int32_t* ids, const int32_t* n_ids,
                               float* out, cudaStream_t s, int nq, float* lse, int warm) {
  switch (L.cfg.n_q_heads / L.cfg.n_kv_heads) {
    case 1: return launch_ac_g<D, 1>(L, fb, q, ids, n_ids, out, s, nq, lse, warm);
    case 2: return launch_ac_g<D, 2>(L, fb, q, ids, n_ids, out, s, nq, lse, warm);
    case 4: return launch_ac_g<D, 4>(L, fb, q, ids, n_ids, out, s, nq, lse, warm);
    case 8: return launch_ac_g<D, 8>(L, fb, q, ids, n_ids, out, s, nq, lse, warm);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_attend(const LayerView& L, const void* q, const int32_t* cells, const int32_t* n_cells, float* out,
                          cudaStream_t s) {
  return L.cfg.head_dim == 128 ? launch_ac_d<128>(L, false, q, cells, n_cells, out, s, 1, nullptr, 0)
                               : launch_ac_d<64>(L, false, q, cells, n_cells, out, s, 1, nullptr, 0);
}

cudaError_t launch_attend_selected(const LayerView& L, const void* q, const int32_t* sel, const int32_t* n_sel,
                                   float* out, cudaStream_t s, int n_queries, float* lse, bool warm) {
  return L.cfg.head_dim == 128 ? launch_ac_d<128>(L, true, q, sel, n_sel, out, s, n_queries, lse, warm)
                               : launch_ac_d<64>(L, true, q, sel, n_sel, out, s, n_queries, lse, warm);
}

// Cluster size and cells per CTA for a configuration, plus the kernel attributes they
// need; called once per context, outside any stream capture.
template <int D, int G>
static cudaError_t plan_ac_g(const qsa_config& c, int* cluster, int* lc) {
  const int mc = max_cells_of(c);
  for (int cs : {16, 8}) {
    const int l = (mc + cs - 1) / cs;
    const size_t smem = AcSmem<D, G>::bytes(l, cs);
    if (smem > 220 * 1024 || AcSmem<D, G>::lp(l) > 256) continue;
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
    e = cs == 16 ? cudaOccupancyMaxActiveClusters(&active, attn_cluster_kernel<D, G, 16, true, false>, &cfg)
                 : cudaOccupancyMaxActiveClusters(&active, attn_cluster_kernel<D, G, 8, true, false>, &cfg);
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
unsigned long long g_noalloc_ctx[kMaxDevices];  // id of the context the address belongs to

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (0 if it cannot be read). A device
// reset or a primary-context teardown gives the device a new context with a new id, and
// the array a new address in it.
unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
    looked_up = true;
  }
  CUcontext c = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&c) != CUDA_SUCCESS || !c || get_id(c, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Once per device (and again if the device's context was replaced since), with that
// device current: look up the array's device address (host code cannot use the symbol
// itself, which is only a host-side stand-in).
cudaError_t noalloc_setup(void** addr, int* n_sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  // 0 when no context is current on this thread yet (the lookup below makes it current)
  const unsigned long long ctx_id = current_ctx_id();
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[dev] || ctx_id == 0 || g_noalloc_ctx[dev] != ctx_id) {
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_sms[dev] = sms;
    g_noalloc_addr[dev] = p;
    g_noalloc_ctx[dev] = current_ctx_id();
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
