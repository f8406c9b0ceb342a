// tile_math.cuh -- per-element helpers shared by the tcgen05 kernels:
// approximate tanh / SiLU and the integer time-bucket search.
#pragma once
#include <cstdint>

namespace hstu {

__device__ __forceinline__ float tanh_approx(float x) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(x));
  return t;
}

__device__ __forceinline__ float silu_precise(float x) { return x / (1.0f + __expf(-x)); }

// bucket(|dt|) = min(NB-1, floor(ln(max(1,|dt|)) / 0.301)) from the integer
// threshold table thr (thr[k] = smallest |dt| with bucket >= k; INT64_MAX
// past NB-1): start from the bucket of the octave's lower end, first_k[e] =
// bucket(2^e), then pass at most three thresholds (ln 2 / 0.301 < 3 buckets
// per octave).
__device__ __forceinline__ int time_bucket(long long dt, const long long* thr,
                                           const signed char* first_k) {
  unsigned long long a = dt < 0 ? 0ull - static_cast<unsigned long long>(dt)
                                : static_cast<unsigned long long>(dt);
  if (a < 1ull) a = 1ull;
  int e = 63 - __clzll(static_cast<long long>(a));
  if (e > 62) e = 62;
  int k = first_k[e];
  // Clamp below the INT64_MAX sentinels that close the table after bucket NB-1.
  const long long aa = static_cast<long long>(a > 0x7FFFFFFFFFFFFFFEull ? 0x7FFFFFFFFFFFFFFEull : a);
  k += (aa >= thr[k + 1]);
  k += (aa >= thr[k + 1]);
  k += (aa >= thr[k + 1]);
  return k;
}

}  // namespace hstu
