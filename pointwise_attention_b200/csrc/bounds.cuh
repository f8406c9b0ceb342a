// bounds.cuh -- index checks of the HSTU_DEBUG_BOUNDS build.
//
// In a build with -DHSTU_DEBUG_BOUNDS every data-derived global index, TMA
// row coordinate and workspace slot of the kernels passes through checked():
// an index outside [0, n) sets the bounds bit of the workspace status word,
// records the first failing site and index (status words 6 and 7) and is
// replaced by 0, so the access stays in bounds and nothing traps.  In the
// normal build checked() returns its index unchanged and compiles away.
#pragma once
#include "internal.h"

namespace hstu {

#ifdef HSTU_DEBUG_BOUNDS
constexpr bool kDebugBounds = true;
#else
constexpr bool kDebugBounds = false;
#endif

// Check sites (status word 6 holds the first one that failed).
enum BoundsSite {
  BS_FWD_TS = 1, BS_FWD_TMA_Q, BS_FWD_TMA_KV, BS_FWD_ROW,
  BS_BWD_TS = 10, BS_BWD_TMA_Q, BS_BWD_TMA_K, BS_BWD_ROW,
  BS_CAND_TS = 20, BS_CAND_TMA, BS_CAND_ROW, BS_CAND_CNT,
  BS_PROJ_TMA = 30, BS_SIMT_TS = 40
};

static __device__ __noinline__ void report_bounds(int* status, int site, long long idx) {
  if (!status) return;
  atomicOr(status, kStatusBounds);
  if (atomicCAS(status + 6, 0, site) == 0) status[7] = static_cast<int>(idx);
}

template <typename I>
__device__ __forceinline__ I checked(int* status, I i, long long n, int site) {
  if (kDebugBounds && !(static_cast<long long>(i) >= 0 && static_cast<long long>(i) < n)) {
    report_bounds(status, site, static_cast<long long>(i));
    return I(0);
  }
  return i;
}

}  // namespace hstu
