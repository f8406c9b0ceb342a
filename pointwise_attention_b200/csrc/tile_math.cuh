// tile_math.cuh -- per-element helpers shared by the tcgen05 kernels:
// approximate tanh / SiLU, bf16x2 arithmetic and the integer time-bucket
// searches.
#pragma once
#include <cuda_bf16.h>

#include <cstdint>

#include "internal.h"   // kMaxBuckets

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

// ------------------------------------------------------------ time-bias plans
// Plan of one row's time bias over a 32-column block, chosen warp-uniformly.
// When the block's column timestamps ascend, every |dt| is below 2^31 and dt
// keeps one sign, each row's bucket moves monotonically along its 32 columns,
// by `spread` buckets at most over the warp: TB_CONST (spread 0), TB_SPLIT (1)
// and TB_MULTI (2 or 3) take per-row split columns found by bisection and add
// the time bias as one more bf16 pair on the packed path.  Otherwise every
// element looks its bucket up: TB_GEN32 on 32-bit differences, TB_GEN64 when
// the span reaches 2^31.  TB_NONE: no time table (or a block that is all
// masked).
enum { TB_NONE = 0, TB_CONST = 1, TB_SPLIT = 2, TB_MULTI = 3, TB_GEN32 = 4, TB_GEN64 = 5 };
// A kernel's own per-element kind: the buckets precomputed per element (one
// byte each) for the blocks nearest the diagonal.
constexpr int TB_BYTES = 6;

// The bucket of column 0 is k_a; from column s[t] on it is t + 1 buckets
// further (down when dt falls along the columns, up when it rises); 32: never.
// v[t]: the half bias of the t-th bucket as a (v, v) pair; t_ab = (v0, v1).
struct TimePlan {
  int k_a;
  int s[3];
  uint32_t v[4];
  uint32_t t_ab;
};

// Columns c = 0..31 with ts32[c] - my32 < th (dt rising along ascending
// columns, dt >= 0): a fixed five-step bisection, then the last column.
__device__ __forceinline__ int count_below_up(const uint32_t* ts32, uint32_t my32, uint32_t th) {
  int pos = 0;
#pragma unroll
  for (int step = 16; step > 0; step >>= 1)
    if (ts32[pos + step - 1] - my32 < th) pos += step;
  return pos + static_cast<int>(ts32[pos] - my32 < th);
}

// Columns with my32 - ts32[c] >= th (dt falling along ascending columns).
__device__ __forceinline__ int count_at_least_dn(const uint32_t* ts32, uint32_t my32, uint32_t th) {
  int pos = 0;
#pragma unroll
  for (int step = 16; step > 0; step >>= 1)
    if (my32 - ts32[pos + step - 1] >= th) pos += step;
  return pos + static_cast<int>(my32 - ts32[pos] >= th);
}

// Tab: the bucket tables in shared memory, with oct(), thr32() and rabt()
// (half time bias per bucket).
template <class Tab>
__device__ __forceinline__ uint32_t bias_pair(const Tab& tt, int k) {
  const float v = tt.rabt()[k];
  return pack_bf16x2(v, v);
}

// The plan's shape: k_a, the split columns and the plan kind, which depend on
// the timestamps only (not on the head's bias table).
//
// Rows at my_ts against later columns (timestamps in [cmin, cmax], low 32
// bits in ts32): dt = t_column - my_ts rises along the columns, so the bucket
// climbs from k_a.
template <class Tab>
__device__ __forceinline__ int plan_shape_up(TimePlan& p, long long my_ts, long long cmin,
                                             long long cmax, bool asc, const uint32_t* ts32,
                                             const Tab& tt) {
  const long long dlo = cmin - my_ts, dhi = cmax - my_ts;
  const bool fast = dhi < 0x7FFFFFFFll && dlo > -0x7FFFFFFFll;
  const bool mono = fast && asc && dlo >= 0;
  int k_b = 0;
  p.k_a = 0;
  p.s[0] = p.s[1] = p.s[2] = 32;
  if (mono) {
    p.k_a = bucket32(static_cast<uint32_t>(dlo), tt.oct());
    k_b = bucket32(static_cast<uint32_t>(dhi), tt.oct());
  }
  if (__all_sync(0xffffffffu, mono)) {
    const int spread = __reduce_max_sync(0xffffffffu, static_cast<unsigned>(k_b - p.k_a));
    if (spread <= 3) {
      const uint32_t my32 = static_cast<uint32_t>(my_ts);
#pragma unroll
      for (int t = 0; t < 3; ++t) {
        // columns still in buckets <= k_a + t: dt < thr[k_a + t + 1]
        const int kt = p.k_a + t + 1;
        if (t < spread)
          p.s[t] = count_below_up(ts32, my32, kt < kMaxBuckets ? tt.thr32()[kt] : 0xFFFFFFFFu);
      }
      return spread == 0 ? TB_CONST : spread == 1 ? TB_SPLIT : TB_MULTI;
    }
  }
  return __all_sync(0xffffffffu, fast) ? TB_GEN32 : TB_GEN64;
}

// Rows at my_ts against earlier columns: dt = my_ts - t_column falls along
// the columns, so the bucket drops from k_a.
template <class Tab>
__device__ __forceinline__ int plan_shape_dn(TimePlan& p, long long my_ts, long long cmin,
                                             long long cmax, bool asc, const uint32_t* ts32,
                                             const Tab& tt) {
  const long long dhi = my_ts - cmin, dlo = my_ts - cmax;
  const bool fast = dhi < 0x7FFFFFFFll && dlo > -0x7FFFFFFFll;
  const bool mono = fast && asc && dlo >= 0;
  int k_b = 0;
  p.k_a = 0;
  p.s[0] = p.s[1] = p.s[2] = 32;
  if (mono) {
    p.k_a = bucket32(static_cast<uint32_t>(dhi), tt.oct());
    k_b = bucket32(static_cast<uint32_t>(dlo), tt.oct());
  }
  if (__all_sync(0xffffffffu, mono)) {
    const int spread = __reduce_max_sync(0xffffffffu, static_cast<unsigned>(p.k_a - k_b));
    if (spread <= 3) {
      const uint32_t my32 = static_cast<uint32_t>(my_ts);
#pragma unroll
      for (int t = 0; t < 3; ++t) {
        // columns still in buckets >= k_a - t: dt >= thr[k_a - t]
        const int kt = p.k_a - t;
        if (t < spread && kt > 0) p.s[t] = count_at_least_dn(ts32, my32, tt.thr32()[kt]);
      }
      return spread == 0 ? TB_CONST : spread == 1 ? TB_SPLIT : TB_MULTI;
    }
  }
  return __all_sync(0xffffffffu, fast) ? TB_GEN32 : TB_GEN64;
}

// The plan's values: the head's half bias of the buckets it passes, as pairs
// (UP: buckets rise from k_a, else they fall).  Kinds other than TB_CONST,
// TB_SPLIT and TB_MULTI need none.
template <bool UP, class Tab>
__device__ __forceinline__ void plan_values(TimePlan& p, int tb, const Tab& tt) {
  if (tb < TB_CONST || tb > TB_MULTI) return;
  const int n = tb == TB_CONST ? 1 : tb == TB_SPLIT ? 2 : 4;
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const int k = UP ? min(p.k_a + min(t, n - 1), kMaxBuckets - 1) : max(p.k_a - min(t, n - 1), 0);
    p.v[t] = bias_pair(tt, k);
  }
  p.t_ab = __byte_perm(p.v[0], p.v[1], 0x7610);
}

// A plan's shape in one word: k_a (7 bits), the three split columns (6 bits
// each, 0..32) and the kind (3 bits).
__device__ __forceinline__ uint32_t plan_word(const TimePlan& p, int tb) {
  return static_cast<uint32_t>(p.k_a) | (static_cast<uint32_t>(p.s[0]) << 7) |
         (static_cast<uint32_t>(p.s[1]) << 13) | (static_cast<uint32_t>(p.s[2]) << 19) |
         (static_cast<uint32_t>(tb) << 25);
}

__device__ __forceinline__ int plan_unword(TimePlan& p, uint32_t w) {
  p.k_a = static_cast<int>(w & 127u);
  p.s[0] = static_cast<int>((w >> 7) & 63u);
  p.s[1] = static_cast<int>((w >> 13) & 63u);
  p.s[2] = static_cast<int>((w >> 19) & 63u);
  return static_cast<int>((w >> 25) & 7u);
}

// The plan's half bias of column c (the buckets passed before it).
__device__ __forceinline__ uint32_t plan_value(const TimePlan& p, int c) {
  return c >= p.s[2] ? p.v[3] : c >= p.s[1] ? p.v[2] : c >= p.s[0] ? p.v[1] : p.v[0];
}

// Half time bias pair of columns 2i, 2i+1 under a TB_CONST / SPLIT / MULTI plan.
template <int TB>
__device__ __forceinline__ uint32_t plan_pair(const TimePlan& p, int i) {
  if (TB == TB_CONST) return p.v[0];
  if (TB == TB_SPLIT) return (2 * i + 1 < p.s[0]) ? p.v[0] : ((2 * i < p.s[0]) ? p.t_ab : p.v[1]);
  return __byte_perm(plan_value(p, 2 * i), plan_value(p, 2 * i + 1), 0x7610);
}

// Buckets of columns 2i, 2i+1 from a row's 32 bucket bytes (8 words); the
// 7-bit mask keeps any word in range of the bucket tables (rows past a
// sequence's end read words they were not written for, and mask the result).
__device__ __forceinline__ int2 byte_bucket_pair(const uint32_t* w8, int i) {
  const uint32_t w = w8[i >> 1] >> (16 * (i & 1));
  return make_int2(static_cast<int>(w & 0x7Fu), static_cast<int>((w >> 8) & 0x7Fu));
}

// Buckets of columns 2i, 2i+1 on the per-element 32-bit path (|dt| < 2^31),
// from the low 32 bits of the columns' and the row's timestamps.
template <class Tab>
__device__ __forceinline__ int2 gen_bucket_pair(const uint32_t* ts32, int i, uint32_t my32,
                                                const Tab& tt) {
  const uint2 t2 = *reinterpret_cast<const uint2*>(ts32 + 2 * i);
  const int d0 = static_cast<int>(t2.x - my32), d1 = static_cast<int>(t2.y - my32);
  return make_int2(bucket32(static_cast<uint32_t>(d0 < 0 ? -d0 : d0), tt.oct()),
                   bucket32(static_cast<uint32_t>(d1 < 0 ? -d1 : d1), tt.oct()));
}

}  // namespace hstu
