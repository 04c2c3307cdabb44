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
// stopping as soon as every key with the current prefix is needed. When the scan's 11-bit
// histogram gives the bin of the K-th key, the CTAs send the keys at or above that bin to
// CTA 0, which refines inside the bin on its own (gather_finish); otherwise every CTA takes
// part in every pass as follows. CTA r of the cluster owns blocks
// [r*kTopkThreads*P, (r+1)*kTopkThreads*P), thread t the P consecutive blocks starting at
// t*P, held in registers (P <= V: the smallest power of two that spreads the layer's
// capacity over the whole cluster). Per pass, each CTA histograms its keys in shared memory and
// pushes the histogram into every CTA's inbox with distributed-shared-memory stores; after
// one cluster barrier each CTA adds the histograms from its own memory. The output
// position of a selected block is the number of keys above the threshold before it plus
// min(need, ties before it); the per-CTA counts follow from the pushed histograms, so one
// packed prefix scan inside the CTA gives every position; ties are taken in block order.
// No CTA reads another's shared memory.
#pragma once

#include <cooperative_groups.h>

#include "qsa_device.cuh"
#include "qsa_sm100.cuh"
#include "qsa_timeline.cuh"

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

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// The same prefix sum with one barrier: warp scans, warp totals through s_warp, and each
// warp adds the totals of the warps before it with shuffles. The caller keeps s_warp
// unwritten until every thread has returned (a barrier lies between two calls).
__device__ __forceinline__ uint32_t cta_exclusive_scan_1(uint32_t v, uint32_t* s_warp, uint32_t* total) {
  constexpr int W = kThreads / 32;
  static_assert(W <= 32, "one warp total per lane");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  const uint32_t w = lane < W ? s_warp[lane] : 0u;
  uint32_t before = lane < warp ? w : 0u, all = w;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    before += __shfl_xor_sync(0xffffffffu, before, off);
    all += __shfl_xor_sync(0xffffffffu, all, off);
  }
  *total = all;
  return before + x - v;
}

enum { kStale = 0, kAll = 1, kTopK = 2 };

struct Result {
  int status;    // kStale: pooled cache behind the context (nothing selected)
                 // kAll: n_blocks <= K, every block is selected (emit not called)
                 // kTopK: K blocks emitted
  int n_ctx;
  int n_blocks;
};

// The selection's finish once the histogram has given the bin b1 holding the K-th largest
// key (prefix = b1's key bits, mask = its 11 bits, need = K minus the keys above b1):
// every CTA sends its keys at or above b1 with their blocks (in block order) and its count
// into CTA 0's shared memory with asynchronous remote stores that count on an mbarrier
// there; CTA 0 waits on that mbarrier alone (no cluster-wide barrier on the way), refines
// the threshold inside b1 with radix passes on the remaining 21 bits over the gathered
// keys, and emits the selection: keys above the threshold, then ties by lower block. In
// CTA 0, warp r holds CTA r's keys (lane l the items l + 32k), so the positions in block
// order come from warp ballots plus one exchange of per-warp counts; one warp scans each
// pass's digit counts. A CTA with more candidates than its
// region holds (a table of near-ties) sends an overflow mark instead, and CTA 0 then runs
// the same passes over every block's score read from memory, kThreads * 8 at a time.
// Every CTA arrives on a final cluster barrier once its data is in place (CTA 0: once it
// has everything) and waits on it before leaving, so no CTA exits while stores into its
// shared memory may still arrive.
template <int V, class ClearHist, class Emit>
__device__ __forceinline__ Result gather_finish(DevState* st, const float* __restrict__ scores, const uint32_t (&key)[V],
                                             uint32_t valid, int base, int n, int n_blocks, uint32_t prefix,
                                             uint32_t mask, uint32_t need, uint64_t* gather_bar, void* region,
                                             uint32_t* s_hist, uint32_t* s_warp, uint32_t* s_ctl, ClearHist&& clear_hist,
                                             Emit&& emit) {
  constexpr uint32_t kCap = 256;               // candidates per source CTA in CTA 0's region
  constexpr uint32_t kOverflow = 0xffffffffu;
  constexpr int kP = 8;                        // items per thread held at once
  constexpr uint32_t kChunk = uint32_t(kThreads) * kP;
  static_assert(kCap == 32 * kP && kThreads / 32 == kCS, "warp r holds CTA r's region, 8 items per lane");
  __shared__ uint32_t s_cnt[kCS];
  uint2* s_cand = static_cast<uint2*>(region);  // [kCS][kCap]
  const int rank = int(cg::this_cluster().block_rank());
  const int tid = threadIdx.x;

  // this CTA's candidates: keys at or above b1, in block order
  uint32_t c = 0;
#pragma unroll
  for (int j = 0; j < V; ++j) c += ((valid >> j) & 1u) && key[j] >= prefix;
  uint32_t tot;
  uint32_t off = cta_exclusive_scan_1(c, s_warp, &tot);  // a barrier since the last s_warp use
  if (rank == 1 && tid == 0) QSA_TL(st, kTlTopk3, 2);  // candidate offsets known
  cluster_wait();  // every CTA of the cluster has started: CTA 0's mbarrier is initialised
  const uint32_t bar0 = sm100::cluster_addr(gather_bar, 0);
  const bool fits = tot <= kCap;  // uniform in the CTA
  if (fits && c) {
    const uint32_t dst = sm100::cluster_addr(s_cand + size_t(rank) * kCap, 0);
#pragma unroll
    for (int j = 0; j < V; ++j)
      if (((valid >> j) & 1u) && key[j] >= prefix) sm100::st_async_v2(dst + 8u * off++, key[j], uint32_t(base + j), bar0);
  }
  if (tid == 0) {
    sm100::st_async_u32(sm100::cluster_addr(&s_cnt[rank], 0), fits ? tot : kOverflow, bar0);
    sm100::mbar_arrive_expect_tx_remote(bar0, 4u + (fits ? 8u * tot : 0u));
    if (rank == 1) QSA_TL(st, kTlTopk3, 3);  // sent
  }
  // the final cluster barrier only keeps every CTA alive until CTA 0 holds all the data:
  // it orders nothing, so its arrive is relaxed
  if (rank != 0) {
    cluster_arrive_relaxed();
    cluster_wait();
    clear_hist();
    return Result{kTopK, n, n_blocks};  // CTA 0 writes the selection
  }

  // ---------------- CTA 0 ----------------
  if (!sm100::mbar_wait_cluster(gather_bar, 0)) {
    if (tid == 0) record_status(st, QSA_ERR_TIMEOUT);
    (void)sm100::mbar_wait_cluster(gather_bar, 0);  // stores still in flight land before this CTA leaves
    cluster_arrive_relaxed();
    cluster_wait();
    clear_hist();
    return Result{kStale, n, 0};
  }
  cluster_arrive_relaxed();  // every source's data is here: the sources may leave
  if (tid == 0) QSA_TL(st, kTlTopk, kTlA);
#ifdef QSA_TIMELINE
  const long long cyc0 = clock64();
#define QSA_CYC(pt) if (tid == 0) QSA_TL_VALUE(st, kTlCycles, pt, uint32_t(clock64() - cyc0))
#else
#define QSA_CYC(pt) ((void)0)
#endif
  bool over = false;
#pragma unroll
  for (int r = 0; r < kCS; ++r) over |= s_cnt[r] == kOverflow;
  if (!over) {
    // ---- warp r takes CTA r's candidates, lane l its items l + 32k (k < 8), in shared
    // memory where they landed; the candidates' order (block order) is region, then item:
    // k, then lane. The passes hold the keys in registers; the output loop stays rolled
    // and reads them from shared memory again (measured faster than the unrolled loop
    // over the registers). ----
    const int warp = tid >> 5, lane = tid & 31;
    const uint32_t lt = lanemask_lt();
    const uint32_t cnt = s_cnt[warp];
    const uint2* mine = s_cand + size_t(warp) * kCap;
    uint32_t ik[kP], iv = 0;  // the keys, in registers for the passes
#pragma unroll
    for (int k = 0; k < kP; ++k) {
      const uint32_t i = uint32_t(lane + 32 * k);
      ik[k] = i < cnt ? mine[i].x : 0u;
      iv |= (i < cnt ? 1u : 0u) << k;
    }
    if (tid == 0) QSA_TL(st, kTlTopk2, 1);
    QSA_CYC(0);
    // radix passes inside b1 (bits 20..13, 12..5, 4..0); warp 0 scans the digit counts
    for (int shift = 32 - kHistBits - 8;; shift -= 8) {
      const int bits = shift >= 0 ? 8 : 8 + shift;
      shift = shift >= 0 ? shift : 0;
      const uint32_t nb = 1u << bits;
      if (tid < 256) s_hist[tid] = 0u;
      __syncthreads();
#pragma unroll
      for (int k = 0; k < kP; ++k)
        if (((iv >> k) & 1u) && (ik[k] & mask) == prefix) atomicAdd(&s_hist[(ik[k] >> shift) & (nb - 1)], 1u);
      __syncthreads();
      if (warp == 0) {  // lane l: digits nb-1-8l .. nb-8-8l (from the top), 8 per lane
        uint32_t cq[8], sum = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int d = int(nb) - 1 - (8 * lane + q);
          cq[q] = d >= 0 ? s_hist[d] : 0u;
          sum += cq[q];
        }
        uint32_t x = sum;  // inclusive scan of the lane sums
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, x, off);
          if (lane >= off) x += y;
        }
        uint32_t acc = x - sum;  // keys in higher digits than this lane's first
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
      // s_ctl is rewritten only after the next pass's two barriers, which every thread
      // reaches after reading it here
      if (tid == 0) QSA_TL(st, kTlTopk2, 2);  // a pass done
      if (shift == 32 - kHistBits - 8) QSA_CYC(1);
      if (s_ctl[2] == need || shift == 0) break;
    }
    if (tid == 0) QSA_TL(st, kTlTopk, kTlB);
    QSA_CYC(2);
    // output: keys above the threshold, then the first `need` keys at it in block order
    uint32_t g_w = 0, e_w = 0;  // this lane's counts, then the warp's (region's)
#pragma unroll
    for (int k = 0; k < kP; ++k) {
      const uint32_t km = ik[k] & mask;
      g_w += ((iv >> k) & 1u) && km > prefix;
      e_w += ((iv >> k) & 1u) && km == prefix;
    }
    uint32_t ge = (g_w << 16) | e_w;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) ge += __shfl_xor_sync(0xffffffffu, ge, off);
    __syncthreads();  // s_warp's previous readers are done
    if (lane == 0) s_warp[warp] = ge;
    __syncthreads();
    uint32_t before = lane < warp ? s_warp[lane] : 0u;  // regions before this one
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) before += __shfl_xor_sync(0xffffffffu, before, off);
    uint32_t gt_b = before >> 16, eq_b = before & 0xffffu;
#pragma unroll 1
    for (uint32_t i0 = 0; i0 < cnt; i0 += 32) {
      const uint32_t i = i0 + uint32_t(lane);
      const uint2 e = i < cnt ? mine[i] : make_uint2(0u, 0u);
      const uint32_t km = e.x & mask;
      const bool gt = i < cnt && km > prefix, eq = i < cnt && km == prefix;
      const uint32_t bg = __ballot_sync(0xffffffffu, gt), be = __ballot_sync(0xffffffffu, eq);
      const uint32_t g = gt_b + __popc(bg & lt), q = eq_b + __popc(be & lt);
      if (gt) emit(g + min(need, q), int(e.y));
      else if (eq && q < need) emit(g + q, int(e.y));
      gt_b += __popc(bg);
      eq_b += __popc(be);
    }
  } else {
    // ---- a CTA overflowed its region: every block's score from memory, kChunk at a time ----
    const uint32_t n_items = uint32_t(n_blocks);
    const int n_chunks = int((n_items + kChunk - 1) / kChunk);
    uint32_t ik[kP], ib[kP], iv = 0;
    // blocks [ch * kChunk + tid * kP, + kP) into registers: thread order is block order
    auto load = [&](int ch) {
      const uint32_t i0 = uint32_t(ch) * kChunk + uint32_t(tid) * kP;
      iv = 0;
  #pragma unroll
      for (int j = 0; j < kP; ++j) {
        const uint32_t i = i0 + uint32_t(j);
        ik[j] = i < n_items ? score_key(__ldcg(scores + i)) : 0u;
        ib[j] = i;
        if (i < n_items) iv |= 1u << j;
      }
    };
    if (n_chunks == 1) load(0);

    // radix passes inside b1: bits 20..13, 12..5, 4..0
    for (int shift = 32 - kHistBits - 8;; shift -= 8) {
      const int bits = shift >= 0 ? 8 : 8 + shift;
      shift = shift >= 0 ? shift : 0;
      const uint32_t nb = 1u << bits;
      if (tid < 256) s_hist[tid] = 0u;
      __syncthreads();
      for (int ch = 0; ch < n_chunks; ++ch) {
        if (n_chunks > 1) load(ch);
  #pragma unroll
        for (int j = 0; j < kP; ++j)
          if (((iv >> j) & 1u) && (ik[j] & mask) == prefix) atomicAdd(&s_hist[(ik[j] >> shift) & (nb - 1)], 1u);
      }
      __syncthreads();
      // thread t < nb takes digit nb - 1 - t: an inclusive prefix over t counts keys >= digit
      const uint32_t v = tid < int(nb) ? s_hist[nb - 1 - tid] : 0u;
      uint32_t tt;
      const uint32_t excl = cta_exclusive_scan(v, s_warp, &tt);
      if (tid < int(nb) && excl < need && excl + v >= need) {
        s_ctl[0] = nb - 1 - uint32_t(tid);
        s_ctl[1] = excl;
        s_ctl[2] = v;
      }
      __syncthreads();
      need -= s_ctl[1];
      prefix |= s_ctl[0] << shift;
      mask |= (nb - 1) << shift;
      const bool done = s_ctl[2] == need || shift == 0;
      __syncthreads();  // s_ctl and s_hist are rewritten by the next pass
      if (done) break;
    }

    // output: keys above the threshold, and the first `need` keys at it in block order
    uint32_t gt_base = 0, eq_base = 0;
    for (int ch = 0; ch < n_chunks; ++ch) {
      if (n_chunks > 1) load(ch);
      uint32_t c_gt = 0, c_eq = 0;
  #pragma unroll
      for (int j = 0; j < kP; ++j) {
        if (!((iv >> j) & 1u)) continue;
        const uint32_t km = ik[j] & mask;
        c_gt += km > prefix;
        c_eq += km == prefix;
      }
      uint32_t t2;
      const uint32_t before = cta_exclusive_scan((c_gt << 16) | c_eq, s_warp, &t2);
      uint32_t gt_b = gt_base + (before >> 16), eq_b = eq_base + (before & 0xffffu);
  #pragma unroll
      for (int j = 0; j < kP; ++j) {
        if (!((iv >> j) & 1u)) continue;
        const uint32_t km = ik[j] & mask;
        if (km > prefix) {
          emit(gt_b + min(need, eq_b), int(ib[j]));
          ++gt_b;
        } else if (km == prefix) {
          if (eq_b < need) emit(gt_b + eq_b, int(ib[j]));
          ++eq_b;
        }
      }
      gt_base += t2 >> 16;
      eq_base += t2 & 0xffffu;
    }
  }
  QSA_CYC(3);
  if (tid == 0) QSA_TL(st, kTlTopk2, 4);
#undef QSA_CYC
  cluster_wait();
  clear_hist();
  return Result{kTopK, n, n_blocks};
}

// Preconditions: every thread of the cluster executed cluster_arrive_relaxed() and then
// pdl_wait(). Selects among the blocks completed within the first n_ctx - n_back tokens
// (n_back > 0: a query of an earlier token of a multi-query step). Calls
// emit(position, block) once per selected block (kTopK only) and returns the same result
// in every thread of the cluster. Cluster-barrier pairing is complete on return on every
// path.
//
// With `hist` (the 2048-bin histogram of the scores' 11-bit key prefixes that the scan
// filled for exactly these blocks), the bin holding the K-th largest key comes from the
// histogram and gather_finish completes the selection in CTA 0 (gather_bar: its mbarrier,
// initialised for kCS arrivals before the cluster's first arrive). Without it, or if its
// total does not match the block count (a scan whose selection never ran), the radix
// passes below run on every CTA from the top byte. The histogram is cleared for the next
// scan in either case.
//
// Output positions need, for every CTA, how many of its keys lie above the final
// threshold and at it. Each CTA pushes its whole pass histogram to every CTA, so each CTA
// derives every other CTA's counts from its own inbox: no exchange of totals is needed.
template <int V, class Emit>
__device__ __forceinline__ Result cluster_select(DevState* st, const float* __restrict__ scores, uint32_t* hist,
                                                 int k_blocks, int max_blocks, int n_back, uint64_t* gather_bar,
                                                 int fused_max_ctx, Emit&& emit) {
  constexpr int kSlots = 256;                 // digit bins of a pass
  constexpr int kHB = 1 << kHistBits;         // 2048
  static_assert(kThreads * 4 == kHB, "each thread reads 4 histogram bins");
  static_assert(kThreads / 32 == kCS, "one warp per source CTA when reading the inbox");
  static_assert(2 * kCS * kSlots * 4 >= kCS * 256 * 8, "the inbox holds CTA 0's candidate regions");
  __shared__ uint32_t s_hist[kSlots];          // this CTA's histogram of the pass
  // every CTA's histogram, double-buffered by pass; on the histogram path, CTA 0's
  // region for every CTA's candidates instead
  __shared__ __align__(16) uint32_t s_in[2][kCS][kSlots];
  __shared__ uint32_t s_warp[32];
  __shared__ uint32_t s_ctl[4];                // digit, count above the digit, count at the digit
  __shared__ uint32_t s_gt[kCS], s_eq[kCS];    // per CTA: keys above the threshold, keys at it

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = int(cluster.block_rank());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // this thread's P <= V scores (P: the smallest power of two that covers the buffer's
  // capacity max_ctx/4 with every CTA of the cluster, so a shorter context still spreads
  // over all of them), read in the same round trip as the state and the histogram; blocks
  // at or past n_ctx/4 are masked once the state is known. Thread t reads histogram bins
  // [2044 - 4t, 2048 - 4t): thread 0 the top ones.
  int P = 1;
  while (P < V && kCS * kThreads * P < max_blocks) P <<= 1;
  const int base = (rank * kThreads + tid) * P;
  float f[V];
  if (P >= 4 && base + P <= max_blocks) {  // whole 16-byte vectors (base is a multiple of 4)
#pragma unroll
    for (int j = 0; j < V; j += 4) {
      float4 x = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      if (j < P) x = *reinterpret_cast<const float4*>(scores + base + j);
      f[j] = x.x;
      f[j + 1] = x.y;
      f[j + 2] = x.z;
      f[j + 3] = x.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < V; ++j) f[j] = j < P && base + j < max_blocks ? scores[base + j] : 0.0f;
  }
  uint4 h4 = make_uint4(0u, 0u, 0u, 0u);
  if (hist) h4 = *reinterpret_cast<const uint4*>(hist + (kHB - 4 - 4 * tid));
  const int n_state = ld_volatile(&st->n_ctx);
  const int n_pooled = ld_volatile(&st->n_pooled);
#pragma unroll
  for (int j = 0; j < V; ++j) asm volatile("" ::"f"(f[j]));  // keep the loads ahead of the branches
  asm volatile("" ::"r"(h4.x), "r"(h4.y), "r"(h4.z), "r"(h4.w));
  if (rank == 1 && tid == 0) QSA_TL(st, kTlTopk3, 0);  // a source CTA's loads issued
  // fused_max_ctx > 0: the decode step's scan appended token n_state (under the same
  // conditions as here) and scored with it, leaving the state for this kernel to advance
  const bool appended = fused_max_ctx > 0 && n_state >= 0 && n_state < fused_max_ctx &&
                        n_pooled == n_state / kBlock;
  const int n_full = appended ? n_state + 1 : n_state;
  const int n = n_full - n_back;
  const int n_blocks = n / kBlock;
  // clears this CTA's slice of the histogram once every CTA of the cluster has read it
  auto clear_hist = [&]() {
    if (hist && tid < kHB / kCS) hist[rank * (kHB / kCS) + tid] = 0u;
  };
  // advances the state past the appended token, once every CTA has read it (each caller
  // is past a point that every CTA of the cluster reaches only after its state read)
  auto publish = [&]() {
    if (appended && rank == 0 && tid == 0) {
      st->n_ctx = n_full;
      st->n_pooled = n_full / kBlock;
    }
  };
  if (n_pooled != n_state / kBlock || n < 0 || (fused_max_ctx > 0 && !appended)) {  // uniform over the cluster
    if (rank == 0 && tid == 0) record_status(st, QSA_ERR_STATE);
    cluster_wait();
    if (hist) {
      cluster.sync();
      clear_hist();
    }
    return Result{kStale, n, 0};
  }
  if (n_blocks <= k_blocks) {  // uniform over the cluster
    cluster_wait();
    if (hist || appended) {
      cluster.sync();
      clear_hist();
      publish();
    }
    return Result{kAll, n, n_blocks};
  }

  uint32_t key[V];
  uint32_t valid = 0;  // bit j: block base + j exists
#pragma unroll
  for (int j = 0; j < V; ++j) {
    key[j] = score_key(f[j]);
    if (j < P && base + j < n_blocks) valid |= 1u << j;
  }
  if (tid < kSlots) s_hist[tid] = 0;
  if (tid < kCS) s_gt[tid] = 0;

  // the starting prefix: the histogram's bin holding the K-th largest key, if the
  // histogram counts exactly these blocks
  uint32_t prefix = 0, mask = 0, need = uint32_t(k_blocks);
  int first_shift = 24;   // first refinement pass: bits [first_shift, first_shift + 8)
  if (hist) {
    const uint32_t c4 = h4.x + h4.y + h4.z + h4.w;
    uint32_t total;
    __syncthreads();  // s_warp's previous readers are done
    if (rank == 1 && tid == 0) QSA_TL(st, kTlTopk3, 4);  // every warp's loads landed
    const uint32_t above = cta_exclusive_scan_1(c4, s_warp, &total);  // keys in higher bins
    if (total == uint32_t(n_blocks)) {  // uniform: every thread sees the same total
      // bins of this thread from the top: 2047-4t (h4.w), then h4.z, h4.y, h4.x
      const uint32_t hb[4] = {h4.w, h4.z, h4.y, h4.x};
      uint32_t acc = above;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (acc < need && acc + hb[i] >= need) {
          s_ctl[0] = uint32_t(kHB - 1 - 4 * tid - i);
          s_ctl[1] = acc;
        }
        acc += hb[i];
      }
      __syncthreads();
      const uint32_t b1 = s_ctl[0];
      need -= s_ctl[1];
      prefix = b1 << (32 - kHistBits);
      mask = ~0u << (32 - kHistBits);
      first_shift = 32 - kHistBits - 8;  // 13
      if (rank == 1 && tid == 0) QSA_TL(st, kTlTopk3, 1);  // the bin found
    }
  }
  if (first_shift != 24) {  // uniform: the histogram gave the bin; finish in CTA 0
    if (tid == 0) QSA_TL(st, kTlTopk2, 0);  // loads and the histogram's bin done
    const Result r = gather_finish<V>(st, scores, key, valid, base, n, n_blocks, prefix, mask, need, gather_bar,
                                      static_cast<void*>(&s_in[0][0][0]), s_hist, s_warp, s_ctl, clear_hist, emit);
    publish();  // CTA 0 returns after the final cluster barrier
    return r;
  }
  if (tid == 0) QSA_TL(st, kTlTopk2, 0);  // loads and the histogram's bin done
  cluster_wait();  // every CTA of the cluster has started: its shared memory may be written
  if (tid == 0) QSA_TL(st, kTlTopk2, 1);

  // radix passes over the keys that match the prefix, 8-bit digits (the last one narrower)
  for (int pass = 0, shift = first_shift;; ++pass) {
    const int bits = shift >= 0 ? 8 : 8 + shift;
    shift = shift >= 0 ? shift : 0;
    const uint32_t nb = 1u << bits;
    __syncthreads();  // the local histogram is zeroed
#pragma unroll
    for (int j = 0; j < V; ++j)
      if (((valid >> j) & 1u) && (key[j] & mask) == prefix) atomicAdd(&s_hist[(key[j] >> shift) & (nb - 1)], 1u);
    __syncthreads();
    // push slot t into [rank][t] of every CTA's inbox for this pass, and clear it for the
    // next pass. A CTA reuses an inbox buffer two passes later, after a barrier that every
    // CTA passes only once all have finished reading it.
    if (tid < kSlots) {
      const uint32_t mine = s_hist[tid];
      s_hist[tid] = 0;
#pragma unroll
      for (int r = 0; r < kCS; ++r) cluster.map_shared_rank(&s_in[pass & 1][0][0], r)[rank * kSlots + tid] = mine;
    }
    if (pass == 0 && tid == 0) QSA_TL(st, kTlTopk2, 2);  // pass 0 pushed
    cluster.sync();  // release the pushes, acquire every other CTA's
    if (pass == 0 && tid == 0) QSA_TL(st, kTlTopk, kTlA);
    if (pass == 1 && tid == 0) QSA_TL(st, kTlTopk2, 3);
    if (pass == 0) clear_hist();  // every CTA read the histogram before its first push
    const uint32_t(*in)[kSlots] = s_in[pass & 1];
    // thread t < nb takes digit (nb - 1 - t): an inclusive prefix over t counts keys >= digit
    uint32_t v = 0;
    if (tid < int(nb)) {
      const int bin = int(nb) - 1 - tid;
#pragma unroll
      for (int r = 0; r < kCS; ++r) v += in[r][bin];
    }
    uint32_t x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    if (lane == 31 && warp < 8) s_warp[warp] = x;
    __syncthreads();
    if (tid < int(nb)) {
      uint32_t excl = x - v;
#pragma unroll
      for (int w = 0; w < 8; ++w) excl += w < warp ? s_warp[w] : 0u;
      if (excl < need && excl + v >= need) {
        s_ctl[0] = uint32_t(int(nb) - 1 - tid);
        s_ctl[1] = excl;
        s_ctl[2] = v;
      }
    }
    __syncthreads();
    const uint32_t d = s_ctl[0];
    // per source CTA (warp r reads CTA r's row): its keys above the digit in this pass,
    // and at the digit
    {
      const int r = warp;
      uint32_t a = 0;
      for (int b = lane; b < int(nb); b += 32) a += b > int(d) ? in[r][b] : 0u;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
      if (lane == 0) {
        s_gt[r] += a;
        s_eq[r] = in[r][d];
      }
    }
    need -= s_ctl[1];
    prefix |= d << shift;
    mask |= (nb - 1) << shift;
    if (s_ctl[2] == need || shift == 0) break;  // uniform: the threshold is fixed
    shift -= 8;
  }
  __syncthreads();  // s_gt and s_eq complete
  if (tid == 0) QSA_TL(st, kTlTopk, kTlB);

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
  if (tid == 0) QSA_TL(st, kTlTopk2, 4);
  uint32_t gt_before = before >> 16, eq_before = before & 0xffffu;
#pragma unroll
  for (int r = 0; r < kCS; ++r) {
    gt_before += r < rank ? s_gt[r] : 0u;
    eq_before += r < rank ? s_eq[r] : 0u;
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
  publish();  // every CTA passed a cluster barrier after its state read
  return Result{kTopK, n, n_blocks};
}

// Keys each thread holds for a layer of max_blocks blocks: 8, 16 or 32.
inline int keys_per_thread(int max_blocks) {
  return max_blocks <= kCS * kThreads * 8 ? 8 : max_blocks <= kCS * kThreads * 16 ? 16 : 32;
}

}  // namespace sel
}  // namespace qsa
