// tile_math.cuh -- per-element helpers shared by the tcgen05 kernels:
// approximate tanh / SiLU, bf16x2 arithmetic and the integer time-bucket
// searches.
#pragma once
#include <cuda_bf16.h>

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

// bucket(|dt|) for 0 <= |dt| < 2^31 from the packed per-octave table oct[e] =
// {bucket(2^e), thr[k+1], thr[k+2], thr[k+3]} (32-bit thresholds).
__device__ __forceinline__ int bucket32(uint32_t a, const uint4* oct) {
  a = a < 1u ? 1u : a;
  const uint4 o = oct[31 - __clz(static_cast<int>(a))];
  return static_cast<int>(o.x) + (a >= o.y) + (a >= o.z) + (a >= o.w);
}

// ------------------------------------------------------------- bf16x2 pairs
// A pair packs two bf16 values in one 32-bit register, the lower-indexed
// element in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);   // .x (low half) = lo
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ uint32_t hadd2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t tanh2(uint32_t x) {
  uint32_t t;
  asm("tanh.approx.bf16x2 %0, %1;" : "=r"(t) : "r"(x));
  return t;
}

constexpr uint32_t kHalfPair = 0x3F003F00u;   // (0.5, 0.5) in bf16

}  // namespace hstu
