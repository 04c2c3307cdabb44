// Timeline probes of the timeline build (-DQSA_TIMELINE): each decode-step kernel records
// in its layer's workspace (the region after DevState, kTimelineOffset) the first and last value of
// %globaltimer (low 32 bits, ns) that its CTAs reach at named points (entry, return from
// the dependency wait, two phase ends, exit), with 32-bit atomic min/max. The host clears
// the record (min slots to all ones, max slots to zero) and reads it back from the layer
// workspace. The default build compiles every probe to nothing.
#pragma once

#include <stdint.h>

#include "qsa_internal.h"

namespace qsa {

enum { kTlScan = 0, kTlTopk = 1, kTlAttn = 2, kTlTopk2 = 3, kTlAttn2 = 4, kTlScan2 = 5, kTlCycles = 6, kTlTopk3 = 7, kTlScan3 = 8, kTlAttnCyc = 9 };
enum { kTlEntry = 0, kTlWait = 1, kTlA = 2, kTlB = 3, kTlExit = 4 };

#ifdef QSA_TIMELINE
__device__ __forceinline__ void tl_mark(DevState* st, int kernel, int point) {
  uint32_t t;
  asm volatile("mov.u32 %0, %%globaltimer_lo;" : "=r"(t));
  uint32_t* rec = reinterpret_cast<uint32_t*>(reinterpret_cast<unsigned char*>(st) + kTimelineOffset) +
                  (kernel * kTimelinePoints + point) * 2;
  atomicMin(rec, t);
  atomicMax(rec + 1, t);
}
// records a value (a count, not a time) in a slot, as its min and max
__device__ __forceinline__ void tl_value(DevState* st, int kernel, int point, uint32_t v) {
  uint32_t* rec = reinterpret_cast<uint32_t*>(reinterpret_cast<unsigned char*>(st) + kTimelineOffset) +
                  (kernel * kTimelinePoints + point) * 2;
  atomicMin(rec, v);
  atomicMax(rec + 1, v);
}
#define QSA_TL(st, kernel, point) ::qsa::tl_mark((st), (kernel), (point))
#define QSA_TL_VALUE(st, kernel, point, v) ::qsa::tl_value((st), (kernel), (point), (v))
#else
#define QSA_TL(st, kernel, point) ((void)0)
#define QSA_TL_VALUE(st, kernel, point, v) ((void)0)
#endif

}  // namespace qsa
