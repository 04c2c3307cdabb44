// Device helpers shared by the kernels: programmatic-dependent-launch controls, the
// status word, warp reductions and a launch wrapper.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "qsa_internal.h"

namespace qsa {

// Wait until the previous kernel on the stream has completed and its writes are
// visible. Every kernel executes this on every path before it exits, so completion
// stays transitive along the stream even when a kernel starts early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Allow the next kernel on the stream to begin launching (its blocks still wait in
// pdl_wait() for this grid to complete before reading anything it wrote).
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Split cluster barrier: every thread arrives early (no memory ordering) and waits
// right before its CTA first writes another CTA's shared memory, which is then known
// to have started. Each thread alternates arrive and wait, like any cluster barrier.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

// Rotation pair of element e of an indexer key or query whose first R dims are rotary
// (Part 10, section "QSA indexer": RoPE at the block position). NeoX style pairs
// (i, i + R/2), interleaved (GPT-J) style pairs (2i, 2i + 1); pair i turns by the angle
// pos * base^(-2i/R). Output e = x[e] * cos + sign * x[partner] * sin, so the first element
// of a pair takes sign -1 and the second +1. Elements e >= R are not rotated (freq < 0).
struct RopeSlot {
  int partner;
  float sign;
  int freq;
};

__host__ __device__ __forceinline__ RopeSlot rope_slot(int e, int R, bool interleaved) {
  if (e >= R) return RopeSlot{e, 0.0f, -1};
  if (interleaved) return RopeSlot{e ^ 1, (e & 1) ? 1.0f : -1.0f, e >> 1};
  const int half = R / 2;
  return e < half ? RopeSlot{e + half, -1.0f, e} : RopeSlot{e - half, 1.0f, e - half};
}

__device__ __forceinline__ void record_status(DevState* st, int code) {
  atomicCAS(&st->status, 0, code);
}

__device__ __forceinline__ int ld_volatile(const int32_t* p) { return *(volatile const int32_t*)p; }

// Sum over the 32 lanes in a fixed butterfly order (deterministic).
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

// Transposing reduction of V per-lane partial sums (V a power of two <= 32): on return,
// every lane holds the full 32-lane sum of element head_of_lane<V>(lane). It costs
// V-1 + log2(32/V) shuffles instead of V*5. Summation order is fixed.
template <int V>
__device__ __forceinline__ float transpose_reduce(float (&v)[V], int lane) {
#pragma unroll
  for (int half = V / 2, off = 16; half >= 1; half >>= 1, off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? v[i] : v[i + half];
      const float keep = upper ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  float r = v[0];
#pragma unroll
  for (int off = 16 / V; off >= 1; off >>= 1) r += __shfl_xor_sync(0xffffffffu, r, off);
  return r;
}

template <int V>
__device__ __forceinline__ int head_of_lane(int lane) {
  // bits [4 .. 5-log2(V)] of the lane, bit 4 most significant
  return V == 1 ? 0 : (lane >> (5 - __builtin_ctz(V))) & (V - 1);
}

// Sum, over the V distinct elements left by transpose_reduce<V>, of one value per
// element (lanes holding the same element must hold the same value).
template <int V>
__device__ __forceinline__ float sum_over_heads(float x) {
#pragma unroll
  for (int off = 16; off >= 32 / V; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

// Preferred shared-memory carveout of every kernel of the decode step: the largest shared
// memory configuration. The scan, selection and attention kernels overlap through
// programmatic dependent launch, and CTAs of different kernels can share an SM only when
// the SM's configuration holds both; the largest one lets a scan CTA start beside an
// attention CTA (or a selection CTA beside a scan CTA) instead of waiting for it to exit.
constexpr int kCarveoutMaxShared = 100;  // percent (cudaSharedmemCarveoutMaxShared)

// Launch with programmatic stream serialization (PDL) and an optional cluster shape.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, int cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (cluster_x > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = cluster_x;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace qsa
