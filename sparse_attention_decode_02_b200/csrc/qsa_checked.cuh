// Bounds guard of the checked build (-DQSA_CHECKED, the stand-in for a memory sanitizer):
// a false condition records QSA_ERR_BAD_INDEX in the layer status and the guarded access is
// skipped; nothing traps. In the default build the guard is the constant true.
#pragma once

#include "qsa_device.cuh"

#ifdef QSA_CHECKED
#define QSA_GUARD(st, cond) ((cond) ? true : (::qsa::record_status((st), QSA_ERR_BAD_INDEX), false))
#else
#define QSA_GUARD(st, cond) true
#endif
