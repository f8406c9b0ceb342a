// bwd_sm100.cu -- bf16 backward of HSTU causal pointwise aggregated attention
// on sm_100a with tcgen05 MMAs (TMEM accumulators, TMA-staged operands).
//
// With x = S + bias, P' = SiLU(x) and dS' = (dO . v_j) SiLU'(x) (the 1/N
// factor of the forward is applied once to every output in fp32):
//   dV_j = 1/N sum_i P'_ij dO_i        dK_j = 1/N sum_i dS'_ij q_i
//   dQ_i = 1/N sum_j dS'_ij k_j        d_rab[h][idx(i,j)] += dS'_ij / N
// where SiLU'(x) = sigma(x) (1 + x (1 - sigma(x))) and sigma(x) comes from the
// same tanh as SiLU: sigma(x) = (1 + tanh(x/2)) / 2.  (Chain rule of the
// forward defined by the "HSTU (Generative Recommender)" model card,
// HSTUBlock.forward, with the relative biases of "HSTU Hierarchical
// Sequential Transduction Units", §1 and §3.)
//
// Two kernels, both deterministic (no floating-point atomics on dQ, dK, dV):
//  * hstu_bwd_dkdv_sm100 -- one CTA per (sequence, key tile n of 128 keys,
//    head).  It walks the query tiles m >= n in sub-tiles of 64 queries
//    x = 0, 1, ...: S^T = K Q_x^T and dA^T = V dO_x^T go to TMEM buffer x % 2;
//    the epilogue writes P'^T and dS'^T (bf16) over them; dV += P'^T dO_x
//    and dK += dS'^T Q_x accumulate in TMEM.
//  * hstu_bwd_dq_sm100 -- one CTA per (sequence, query tile m, head), key
//    sub-tiles x of 64 keys over tiles 0..m: S = Q K_x^T, dA = dO V_x^T, the
//    epilogue writes dS' over dA and sums dS' along the position diagonals
//    and per time bucket (the bias gradients); dQ += dS' K_x accumulates.
// In both, two groups of eight epilogue warps take the even and the odd
// sub-tiles, so one group's epilogue runs while the tensor core works on the
// other's sub-tile: with S and dA double-buffered at 64 columns each, TMEM
// (512 columns) still holds the 128-column accumulators.
//
// Roles: warp 0 TMA (the resident 128-row tiles, then 3-stage rings of
// 64-row sub-tiles); warps 2..17 the epilogue; MMAs issued by one thread in
// each of warps 1, 18 and 19, one per independent chain: a tcgen05.mma costs
// its issuing thread about 80-110 cycles, longer than a 128 x 64 x 16 step
// takes on the tensor core, so the chains are issued in parallel.

#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>

#include "bounds.cuh"
#include "internal.h"
#include "ptx.cuh"
#include "tile_math.cuh"

namespace hstu {
namespace {

constexpr int kThreads = 640;
constexpr int kEpi = 512;
constexpr int kWarpB = 18;                   // second MMA issuer
constexpr int kWarpC = 19;                   // third MMA issuer
constexpr int kHalf = 16384;                 // 128 rows x 64 bf16
constexpr int kTile = 2 * kHalf;             // 128 x 128 bf16
constexpr int kTmemCols = 512;

__device__ __forceinline__ void set_status(int* status, int bit) {
  if (status) atomicOr(status, bit);
}

// From hx = (S + bias)/2 and t = tanh(hx):
//   sigma(x) = (1 + t)/2,  P' = SiLU(x) = hx (1 + t),
//   SiLU'(x) = sigma(x) (1 + x (1 - sigma(x))) = sigma(x) (1 + hx (1 - t)).
__device__ __forceinline__ float silu_grad_h(float hx, float t) {
  const float sg = fmaf(t, 0.5f, 0.5f);
  return sg * fmaf(hx, 1.0f - t, 1.0f);
}

// Per-warp staging of one 32 x 32 block: 63 position-bias diagonals (fp32,
// halved) and the 32 column timestamps (also their low 32 bits, whose
// differences are exact while |dt| < 2^31).
struct Stage {
  float w[64];
  long long ts[32];
  uint32_t ts32[32];
  // bf16 pairs of neighbouring diagonals for the packed path: (w[k], w[k+1])
  // in the dK/dV kernel, (w[k], w[k-1]) in the dQ kernel
  uint32_t wpk[64];
};

// Stage the block's 32 column timestamps (lane c holds column c's) for the
// per-element paths.
__device__ __forceinline__ void stage_time(Stage* stg, int lane, long long pt) {
  stg->ts[lane] = pt;
  stg->ts32[lane] = static_cast<uint32_t>(pt);
}

constexpr uint32_t kOne2 = 0x3F803F80u;     // (1, 1)
constexpr uint32_t kNegOne2 = 0xBF80BF80u;  // (-1, -1)

// Packed P' and dS' of an element pair from hx = S/2 + bias/2 (bf16 pairs):
// t = tanh(hx), P' = hx (1 + t), SiLU'(x) = (1 + t)/2 (1 + hx (1 - t)).
__device__ __forceinline__ uint32_t dsilu_pair(uint32_t hx, uint32_t t, uint32_t da) {
  const uint32_t sg = hfma2(t, kHalfPair, kHalfPair);
  const uint32_t q = hfma2(hx, hfma2(t, kNegOne2, kOne2), kOne2);
  return hmul2(da, hmul2(sg, q));
}

__device__ __forceinline__ uint32_t pack_u32_pair(uint32_t lo, uint32_t hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(lo), __uint_as_float(hi));
  return *reinterpret_cast<uint32_t*>(&v);
}

// Element hh (0: low, 1: high half) of a bf16 pair, widened to fp32.
__device__ __forceinline__ float bf16_half(uint32_t pair, int hh) {
  return __uint_as_float(hh ? (pair & 0xFFFF0000u) : (pair << 16));
}

// 32 fp32 columns of this warp's TMEM lanes, loaded and packed into bf16
// pairs: every per-element path works from the pairs, so only one block of
// fp32 registers is ever live.
__device__ __forceinline__ void load_pairs(uint32_t taddr, uint32_t (&out)[16]) {
  uint32_t v[32];
  tmem_ld32_nowait(taddr, v);
  tmem_wait_ld_dep(v);
#pragma unroll
  for (int i = 0; i < 16; ++i) out[i] = pack_u32_pair(v[2 * i], v[2 * i + 1]);
}

// The time-bucket tables in shared memory, at fixed offsets from its base.
struct TimeTables {
  const uint8_t* base;
  __device__ __forceinline__ const long long* thr() const;
  __device__ __forceinline__ const signed char* first() const;
  __device__ __forceinline__ const float* rabt() const;    // half time bias per bucket
  __device__ __forceinline__ const uint4* oct() const;
  __device__ __forceinline__ const unsigned* thr32() const;
};

// s_dt[k] += v where flag holds, without a branch.
__device__ __forceinline__ void red_shared_if(const float* p, float v, bool flag) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %2, 0;\n\t@q red.shared.add.f32 [%0], %1;\n\t}" ::"r"(
          smem_u32(p)),
      "f"(v), "r"(static_cast<unsigned>(flag))
      : "memory");
}

// Running (bucket, sum) of one row's dS' on the packed per-element path: the
// sum goes to the shared histogram when a nonzero element changes the bucket.
__device__ __forceinline__ void run_add_packed(int k, float v, int& run_k, float& run_s,
                                               float* s_dt) {
  const bool chg = v != 0.f && k != run_k;
  red_shared_if(s_dt + (run_k < 0 ? 0 : run_k), run_s, chg && run_s != 0.f);
  run_s = chg ? v : run_s + v;
  run_k = chg ? k : run_k;
}

// Running sum of one row's dS' per time bucket on the per-element path: a
// (bucket, sum) pair in registers goes to the shared histogram when the
// bucket changes (sorted timestamps change it rarely along a row).
__device__ __forceinline__ void run_add(int k, float v, int& run_k, float& run_s, float* s_dt) {
  if (v == 0.f) return;
  if (k == run_k) {
    run_s += v;
  } else {
    if (run_k >= 0) atomicAdd(&s_dt[run_k], run_s);
    run_k = k;
    run_s = v;
  }
}

// P'^T and dS'^T of one 32-column chunk of the dK/dV kernel (rows = keys,
// columns = queries); the bias gradients come from the dQ kernel.  MASK:
// the diagonal tile or the sequence's last query tile.
template <bool POS, int TB, bool MASK>
__device__ __forceinline__ void dkv_chunk(const uint32_t (&sp)[16], const uint32_t (&dp)[16],
                                          const Stage* stg, int lane, int r, int c0, bool diag,
                                          int qlim, const TimePlan& tp, long long my_ts,
                                          const TimeTables& tt, uint32_t (&pk)[16],
                                          uint32_t (&dk)[16], const uint32_t* nbw = nullptr) {
  if (TB != TB_GEN64) {
    // bf16x2 arithmetic: P' and dS' are bf16 operands of the next MMAs anyway
    const uint32_t* wp = stg->wpk + 31 - lane;   // pair i: diagonals 2i - lane + 31 (+1)
    const uint32_t my32 = static_cast<uint32_t>(my_ts);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      // half bias pair (position + time), added before S arrives in the chain
      uint32_t hb = POS ? wp[2 * i] : 0u;
      if (TB == TB_GEN32 || TB == TB_BYTES) {
        const int2 kb = TB == TB_BYTES ? byte_bucket_pair(nbw, i) : gen_bucket_pair(stg->ts32, i, my32, tt);
        const uint32_t tb = pack_bf16x2(tt.rabt()[kb.x], tt.rabt()[kb.y]);
        hb = POS ? hadd2(hb, tb) : tb;
      } else if (TB != TB_NONE) {
        hb = POS ? hadd2(hb, plan_pair<TB>(tp, i)) : plan_pair<TB>(tp, i);
      }
      const uint32_t hx = hfma2(sp[i], kHalfPair, hb);
      const uint32_t t = tanh2(hx);
      uint32_t p = hfma2(hx, t, hx);
      uint32_t d = dsilu_pair(hx, t, dp[i]);
      if (MASK) {
        const int c = c0 + 2 * i;
        const uint32_t keep = (((diag && c < r) || c >= qlim) ? 0u : 0x0000FFFFu) |
                              (((diag && c + 1 < r) || c + 1 >= qlim) ? 0u : 0xFFFF0000u);
        p &= keep;
        d &= keep;
      }
      pk[i] = p;
      dk[i] = d;
    }
    return;
  }
  // time spans of 2^31 or more: fp32, 64-bit bucket search
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float p2[2], d2[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int cl = 2 * i + hh;
      const int c = c0 + cl;
      float hb = POS ? stg->w[cl - lane + 31] : 0.f;
      hb += tt.rabt()[time_bucket(stg->ts[cl] - my_ts, tt.thr(), tt.first())];
      const float hx = fmaf(bf16_half(sp[i], hh), 0.5f, hb);
      const float t = tanh_approx(hx);
      float p = fmaf(hx, t, hx);
      float ds = bf16_half(dp[i], hh) * silu_grad_h(hx, t);
      if (MASK && ((diag && c < r) || c >= qlim)) {
        p = 0.f;
        ds = 0.f;
      }
      p2[hh] = p;
      d2[hh] = ds;
    }
    pk[i] = pack_bf16x2(p2[0], p2[1]);
    dk[i] = pack_bf16x2(d2[0], d2[1]);
  }
}

// dS' of one 32-column chunk of the dQ kernel (rows = queries, columns =
// keys), and its bias-gradient sums.  MASK: the diagonal tile, keys past the
// sequence end, or query rows past it (those rows belong to no query of the
// sequence and must not reach the bias gradients).  On the packed paths the
// sums take dS' as rounded to bf16 for the dQ MMA.
template <bool POS, int TB, bool MASK>
__device__ __forceinline__ void dq_chunk(const uint32_t (&sp)[16], const uint32_t (&dp)[16],
                                         const Stage* stg, int lane, int r, int c0, bool diag,
                                         int klim, bool row_ok, const TimePlan& tp,
                                         long long my_ts, const TimeTables& tt, float* win,
                                         int wbase, float* s_dt, uint32_t (&dk)[16], int& run_k,
                                         float& run_s, const uint32_t* nbw = nullptr) {
  // Diagonal sums (row - column = const) of the warp's 32 x 32 block: at
  // column cl lane L reads lane (L + cl) mod 32, so every element with
  // row - cl = L, or L - 32, passes through lane L.
  float dpos = 0.f, dneg = 0.f;
  if (TB != TB_GEN64) {
    const uint32_t* wp = stg->wpk + lane + 31;   // pair i: diagonals lane - 2i + 31 (-1)
    const uint32_t my32 = static_cast<uint32_t>(my_ts);
    // dS' of the row, and of its columns from each split on
    float t_all = 0.f, g1 = 0.f, g2 = 0.f, g3 = 0.f;
    // sums of diagonals lane - 1 and lane - 33, the next lane's to take
    float dpos1 = 0.f, dneg1 = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      // half bias pair (position + time), added before S arrives in the chain
      uint32_t hb = POS ? wp[-2 * i] : 0u;
      int2 kb = make_int2(0, 0);
      if (TB == TB_GEN32 || TB == TB_BYTES) {
        kb = TB == TB_BYTES ? byte_bucket_pair(nbw, i) : gen_bucket_pair(stg->ts32, i, my32, tt);
        const uint32_t tb = pack_bf16x2(tt.rabt()[kb.x], tt.rabt()[kb.y]);
        hb = POS ? hadd2(hb, tb) : tb;
      } else if (TB != TB_NONE) {
        hb = POS ? hadd2(hb, plan_pair<TB>(tp, i)) : plan_pair<TB>(tp, i);
      }
      const uint32_t hx = hfma2(sp[i], kHalfPair, hb);
      uint32_t d = dsilu_pair(hx, tanh2(hx), dp[i]);
      if (MASK) {
        const int c = c0 + 2 * i;
        const uint32_t keep =
            (((diag && c > r) || c >= klim || !row_ok) ? 0u : 0x0000FFFFu) |
            (((diag && c + 1 > r) || c + 1 >= klim || !row_ok) ? 0u : 0xFFFF0000u);
        d &= keep;
      }
      dk[i] = d;
      const float v0 = __uint_as_float(d << 16), v1 = __uint_as_float(d & 0xFFFF0000u);
      if (POS) {
        // the pair of row (lane + 2i) mod 32: its low element lies on this
        // lane's diagonal, its high one on the next lower diagonal
        const uint32_t pr = __shfl_sync(0xffffffffu, d, (lane + 2 * i) & 31);
        const float lo = __uint_as_float(pr << 16), hi = __uint_as_float(pr & 0xFFFF0000u);
        if (lane + 2 * i < 32) {
          dpos += lo;
          dpos1 += hi;
        } else {
          dneg += lo;
          dneg1 += hi;
        }
      }
      if (TB == TB_GEN32 || TB == TB_BYTES) {
        run_add_packed(kb.x, v0, run_k, run_s, s_dt);
        run_add_packed(kb.y, v1, run_k, run_s, s_dt);
      } else if (TB != TB_NONE) {
        t_all += v0 + v1;
        if (TB >= TB_SPLIT) {
          if (2 * i >= tp.s[0]) g1 += v0;
          if (2 * i + 1 >= tp.s[0]) g1 += v1;
        }
        if (TB == TB_MULTI) {
          if (2 * i >= tp.s[1]) g2 += v0;
          if (2 * i + 1 >= tp.s[1]) g2 += v1;
          if (2 * i >= tp.s[2]) g3 += v0;
          if (2 * i + 1 >= tp.s[2]) g3 += v1;
        }
      }
    }
    if (POS) {
      // lane L takes diagonal L from lane L + 1's second sums (lane 31 takes
      // diagonal -1 from lane 0's)
      const float p1 = __shfl_sync(0xffffffffu, dpos1, (lane + 1) & 31);
      const float n1 = __shfl_sync(0xffffffffu, dneg1, (lane + 1) & 31);
      dpos += lane < 31 ? p1 : 0.f;
      dneg += lane < 31 ? n1 : p1;
    }
    if (TB == TB_CONST || TB == TB_SPLIT || TB == TB_MULTI) {
      // The warp's 32 rows (consecutive queries) reach neighbouring buckets:
      // sum each bucket over the warp and let one lane add it to the histogram
      // (per-row running sums instead collide in shared memory: the rows of a
      // warp change bucket together).
      const float b0 = t_all - g1, b1 = g1 - g2, b2 = g2 - g3, b3 = g3;
      const int steps = TB == TB_CONST ? 0 : TB == TB_SPLIT ? 1 : 3;
      const int kmax = __reduce_max_sync(0xffffffffu, static_cast<unsigned>(tp.k_a));
      int kmin = static_cast<int>(__reduce_min_sync(0xffffffffu, static_cast<unsigned>(tp.k_a))) - steps;
      kmin = kmin < 0 ? 0 : kmin;
      // Each bucket's warp sum in fixed point, one integer reduction: the
      // scale 2^(24 - e) (2^e <= the warp's largest |b| < 2^(e+1)) keeps each
      // term below 2^25 and 32 of them inside 30 bits, and rounds each to
      // 2^-25 of that largest term.
      float amax = fmaxf(fmaxf(fabsf(b0), fabsf(b1)), fmaxf(fabsf(b2), fabsf(b3)));
      const unsigned mbits = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
      const int e = static_cast<int>(mbits >> 23) - 127;
      if (mbits != 0u && e > -100 && e < 100) {
        const float scale = __uint_as_float(static_cast<unsigned>(127 + 24 - e) << 23);
        const float unscale = __uint_as_float(static_cast<unsigned>(127 - 24 + e) << 23);
#pragma unroll 1
        for (int kb = kmax; kb >= kmin; --kb) {
          const int t = tp.k_a - kb;
          const float v = t == 0 ? b0 : t == 1 ? b1 : t == 2 ? b2 : t == 3 ? b3 : 0.f;
          const int sum = __reduce_add_sync(0xffffffffu, __float2int_rn(v * scale));
          if (lane == 0 && sum != 0) atomicAdd(&s_dt[kb], static_cast<float>(sum) * unscale);
        }
      } else if (mbits != 0u) {
#pragma unroll 1
        for (int kb = kmax; kb >= kmin; --kb) {
          const int t = tp.k_a - kb;
          float v = t == 0 ? b0 : t == 1 ? b1 : t == 2 ? b2 : t == 3 ? b3 : 0.f;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          if (lane == 0 && v != 0.f) atomicAdd(&s_dt[kb], v);
        }
      }
    }
  } else {
    // time spans of 2^31 or more: fp32, 64-bit bucket search
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float d2[2];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int cl = 2 * i + hh;
        const int c = c0 + cl;
        float hb = POS ? stg->w[lane - cl + 31] : 0.f;
        const int kb = time_bucket(my_ts - stg->ts[cl], tt.thr(), tt.first());
        hb += tt.rabt()[kb];
        const float hx = fmaf(bf16_half(sp[i], hh), 0.5f, hb);
        const float t = tanh_approx(hx);
        float ds = bf16_half(dp[i], hh) * silu_grad_h(hx, t);
        const bool masked = MASK && ((diag && c > r) || c >= klim || !row_ok);
        if (masked) ds = 0.f;
        d2[hh] = ds;
        if (POS) {
          const float v = __shfl_sync(0xffffffffu, ds, (lane + cl) & 31);
          if (lane + cl < 32) dpos += v; else dneg += v;
        }
        if (!masked) run_add(kb, ds, run_k, run_s, s_dt);
      }
      dk[i] = pack_bf16x2(d2[0], d2[1]);
    }
  }
  if (POS) {
    atomicAdd(&win[wbase + lane], dpos);
    if (lane > 0) atomicAdd(&win[wbase + lane - 32], dneg);
  }
}

// ------------------------------------------------------------------ sub-tiles
constexpr int kSub = 8192;                   // 64 rows x 64 bf16 (one 128-byte swizzle span)
constexpr int kSubTile = 2 * kSub;           // 64 rows x 128 bf16
constexpr int kRing = 3;                     // sub-tile stages
constexpr int kGroup = 256;                  // threads of one epilogue group

constexpr uint32_t kIdescN64 = idesc_bf16_f32(128, 64, false, false);  // K-major x K-major, N = 64
constexpr uint32_t kIdescTM = idesc_bf16_f32(128, 128, false, true);   // A TMEM, B MN-major

// D (128 x 64) = A (128 rows x 128, K-major, 64-column halves kHalf apart)
//              * B (64 rows x 128, K-major, halves kSub apart)^T
__device__ __forceinline__ void mma_n64(uint32_t d, uint32_t a_smem, uint32_t b_smem) {
#pragma unroll
  for (int ks = 0; ks < 8; ++ks)
    mma_ss(d, sw128_desc(a_smem + (ks >> 2) * kHalf + (ks & 3) * 32, 16, 1024),
           sw128_desc(b_smem + (ks >> 2) * kSub + (ks & 3) * 32, 16, 1024), kIdescN64,
           ks > 0 ? 1u : 0u);
}

// D (128 x 128) (+)= A (128 x 64 bf16 pairs in TMEM: the warps of column
// half c2 hold reduction indices 32 c2 .. 32 c2 + 31 as pairs in the first 16
// of their own 32 columns, 32 c2 ..) * B (64 rows = reduction index, MN-major,
// 64-column halves kSub apart)
__device__ __forceinline__ void mma_tm64(uint32_t d, uint32_t a_tmem, uint32_t b_smem,
                                         bool accumulate) {
#pragma unroll
  for (int ks = 0; ks < 4; ++ks)
    mma_ts(d, a_tmem + 32u * (ks >> 1) + 8u * (ks & 1), sw128_desc(b_smem + ks * 2048, kSub, 1024),
           kIdescTM, (accumulate || ks > 0) ? 1u : 0u);
}

// Smem offsets shared by both kernels: two resident 128-row tiles, two rings
// of 64-row sub-tiles, per-warp staging, then the tables.
constexpr int kOffT0 = 0;                                 // resident tile 0
constexpr int kOffT1 = kTile;                             // resident tile 1
constexpr int kOffR0 = 2 * kTile;                         // ring 0
constexpr int kOffR1 = kOffR0 + kRing * kSubTile;         // ring 1
constexpr int kOffStage = kOffR1 + kRing * kSubTile;      // 16 warps x Stage
constexpr int kOffWin = kOffStage + 16 * static_cast<int>(sizeof(Stage));   // 2 groups x 2 x 256
constexpr int kOffDT = kOffWin + 4 * 256 * 4;             // 128 fp32
constexpr int kOffThr = kOffDT + 128 * 4;
constexpr int kOffFirst = kOffThr + kThrLen * 8;
constexpr int kOffRabT = kOffFirst + 64;
constexpr int kOffOct = kOffRabT + 128 * 4;               // 32 x uint4
constexpr int kOffThr32 = kOffOct + 32 * 16;
constexpr int kOffBar = kOffThr32 + kMaxBuckets * 4;
constexpr int kNumBars = 24;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmem = kOffMisc + 64 + 1024;
static_assert(kOffStage % 16 == 0 && sizeof(Stage) % 8 == 0, "staging alignment");
static_assert(kOffOct % 16 == 0 && kOffThr % 8 == 0 && kOffBar % 8 == 0, "table alignment");
static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
// TMEM: S (or S^T) of buffer u at 64 u, dA (or dA^T) at 128 + 64 u, the
// accumulators at 256 (dV or dQ) and 384 (dK).
constexpr uint32_t kColS = 0, kColDA = 128, kColAcc0 = 256, kColAcc1 = 384;

__device__ __forceinline__ const long long* TimeTables::thr() const {
  return reinterpret_cast<const long long*>(base + kOffThr);
}
__device__ __forceinline__ const signed char* TimeTables::first() const {
  return reinterpret_cast<const signed char*>(base + kOffFirst);
}
__device__ __forceinline__ const float* TimeTables::rabt() const {
  return reinterpret_cast<const float*>(base + kOffRabT);
}
__device__ __forceinline__ const uint4* TimeTables::oct() const {
  return reinterpret_cast<const uint4*>(base + kOffOct);
}
__device__ __forceinline__ const unsigned* TimeTables::thr32() const {
  return reinterpret_cast<const unsigned*>(base + kOffThr32);
}

// The time-bucket tables of head h in shared memory (epilogue thread et).
__device__ __forceinline__ TimeTables init_tables(const BwdArgs& a, int h, int et, uint8_t* smem) {
  TimeTables tt;
  long long* thr = reinterpret_cast<long long*>(smem + kOffThr);
  signed char* first = reinterpret_cast<signed char*>(smem + kOffFirst);
  float* rabt = reinterpret_cast<float*>(smem + kOffRabT);
  uint4* oct = reinterpret_cast<uint4*>(smem + kOffOct);
  unsigned* thr32 = reinterpret_cast<unsigned*>(smem + kOffThr32);
  if (et >= 0) {
    for (int i = et; i < kThrLen; i += kEpi) thr[i] = a.bt.thr[i];
    if (et < 64) first[et] = a.bt.first_k[et];
    if (et < a.nb) rabt[et] = 0.5f * __ldg(a.rab_time + static_cast<size_t>(h) * a.nb + et);
    if (et < 32) oct[et] = a.bt.oct[et];
    if (et < kMaxBuckets) thr32[et] = a.bt.thr32[et];
  }
  tt.base = smem;
  return tt;
}

// ===================================================================== dK, dV
namespace dkv {
// smem: K (T0), V (T1), Q sub-tiles (R0), dO sub-tiles (R1)
enum {
  B_KVFULL = 0,
  B_QFULL = 1,       // + ring slot
  B_QEMPTY = 4,      // + ring slot (count 2: S^T and dK read Q)
  B_DOFULL = 7,
  B_DOEMPTY = 10,    // count 2: dA^T and dV read dO
  B_SFULL = 13,      // + buffer (count 2: S^T and dA^T)
  B_PFULL = 15,      // + buffer (count kGroup): P'^T, dS'^T written
  B_DVDONE = 17,     // + buffer: dV read P'^T, the S^T columns are free
  B_DKDONE = 19,     // + buffer: dK read dS'^T, the dA^T columns are free
  B_OUT = 21         // count 2: every MMA of both issuers done
};

template <bool POS, bool TIME>
__global__ void __launch_bounds__(kThreads, 1)
    hstu_bwd_dkdv_sm100(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_do,
                        const __grid_constant__ BwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = static_cast<int>(blockIdx.x % static_cast<unsigned>(a.H));
  const int idx = static_cast<int>(blockIdx.x / static_cast<unsigned>(a.H));
  const int n = idx / a.B;                    // key tile; n = 0 has the most query tiles
  const int b = idx % a.B;
  const int s = __ldg(a.offsets + b);
  const int e_ = __ldg(a.offsets + b + 1);
  int n_b = e_ - s;
  if (s < 0 || n_b < 0 || e_ > a.T || n_b > a.max_seq_len || (POS && n_b > a.L)) n_b = 0;
  if (128 * n >= n_b) return;
  const int mt_b = (n_b + 127) / 128;         // query tiles of this sequence
  const int nx = 2 * (mt_b - n);              // query sub-tiles of tiles n .. mt_b-1

  auto bar = [&](int i) { return sbase + kOffBar + 8u * i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

  if (threadIdx.x == 0) {
    for (int i = 0; i <= B_OUT; ++i) {
      uint32_t count = 1;
      if ((i >= B_QEMPTY && i < B_QEMPTY + kRing) || (i >= B_DOEMPTY && i < B_DOEMPTY + kRing) ||
          i == B_SFULL || i == B_SFULL + 1 || i == B_OUT)
        count = 2;
      if (i == B_PFULL || i == B_PFULL + 1) count = kGroup;
      mbar_init(bar(i), count);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sbase + kOffMisc, kTmemCols);
    tmem_relinquish();
  }
  TimeTables tt{};
  if (TIME) tt = init_tables(a, h, (warp >= 2 && warp < kWarpB) ? threadIdx.x - 64 : -1, smem);
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      const int krow = checked(a.status, s + 128 * n, a.T, BS_BWD_TMA_K);
      mbar_arrive_expect_tx(bar(B_KVFULL), 2 * kTile);
      tma_load_3d(sbase + kOffT0, &tm_k, bar(B_KVFULL), 0, h, krow);
      tma_load_3d(sbase + kOffT0 + kHalf, &tm_k, bar(B_KVFULL), 64, h, krow);
      tma_load_3d(sbase + kOffT1, &tm_v, bar(B_KVFULL), 0, h, krow);
      tma_load_3d(sbase + kOffT1 + kHalf, &tm_v, bar(B_KVFULL), 64, h, krow);
      int q_last[kRing] = {-1, -1, -1}, o_last[kRing] = {-1, -1, -1};
      bool ok = true;
      for (int x = 0; x < nx && ok; ++x) {
        const int slot = x % kRing, use = x / kRing;
        const int qrow = checked(a.status, s + 128 * (n + (x >> 1)) + 64 * (x & 1), a.T, BS_BWD_TMA_Q);
        if (use > 0) ok = mbar_wait(bar(B_QEMPTY + slot), (use - 1) & 1, abort_flag);
        if (!ok) break;
        const uint32_t qd = sbase + kOffR0 + slot * kSubTile;
        mbar_arrive_expect_tx(bar(B_QFULL + slot), kSubTile);
        tma_load_3d(qd, &tm_q, bar(B_QFULL + slot), 0, h, qrow);
        tma_load_3d(qd + kSub, &tm_q, bar(B_QFULL + slot), 64, h, qrow);
        q_last[slot] = use;
        if (use > 0) ok = mbar_wait(bar(B_DOEMPTY + slot), (use - 1) & 1, abort_flag);
        if (!ok) break;
        const uint32_t od = sbase + kOffR1 + slot * kSubTile;
        mbar_arrive_expect_tx(bar(B_DOFULL + slot), kSubTile);
        tma_load_3d(od, &tm_do, bar(B_DOFULL + slot), 0, h, qrow);
        tma_load_3d(od + kSub, &tm_do, bar(B_DOFULL + slot), 64, h, qrow);
        o_last[slot] = use;
      }
      if (!ok) {
        set_status(a.status, kStatusTimeout);
        *abort_flag = 1;
        mbar_wait(bar(B_KVFULL), 0, nullptr);
        for (int sl = 0; sl < kRing; ++sl) {
          if (q_last[sl] >= 0) mbar_wait(bar(B_QFULL + sl), q_last[sl] & 1, nullptr);
          if (o_last[sl] >= 0) mbar_wait(bar(B_DOFULL + sl), o_last[sl] & 1, nullptr);
        }
      }
    }
  } else if (warp == 1 || warp == kWarpB) {
    // ------------- MMA issuers: S^T then dV (warp 1); dA^T then dK (warp 18),
    // each one sub-tile ahead with its S^T / dA^T
    if (lane == 0) {
      const bool first = warp == 1;
      bool ok = mbar_wait(bar(B_KVFULL), 0, abort_flag);
      auto ring0 = [&](int x) { return sbase + kOffR0 + (x % kRing) * kSubTile; };
      auto ring1 = [&](int x) { return sbase + kOffR1 + (x % kRing) * kSubTile; };
      // S^T (or dA^T) of sub-tile x into buffer x % 2, once the dV (dK) of
      // sub-tile x - 2 has read that buffer's P'^T (dS'^T)
      auto issue_front = [&](int x) {
        const int slot = x % kRing;
        bool r = mbar_wait(bar((first ? B_QFULL : B_DOFULL) + slot), (x / kRing) & 1, abort_flag);
        if (r && x >= 2)
          r = mbar_wait(bar((first ? B_DVDONE : B_DKDONE) + (x & 1)), ((x - 2) >> 1) & 1, abort_flag);
        if (!r) return false;
        tc_fence_after();
        if (first) {
          mma_n64(tmem + kColS + 64u * (x & 1), sbase + kOffT0, ring0(x));
          mma_commit(bar(B_QEMPTY + slot));
        } else {
          mma_n64(tmem + kColDA + 64u * (x & 1), sbase + kOffT1, ring1(x));
          mma_commit(bar(B_DOEMPTY + slot));
        }
        mma_commit(bar(B_SFULL + (x & 1)));
        return true;
      };
      if (ok) ok = issue_front(0);
      for (int x = 0; x < nx && ok; ++x) {
        if (x + 1 < nx) ok = issue_front(x + 1);
        if (ok) ok = mbar_wait(bar(B_PFULL + (x & 1)), (x >> 1) & 1, abort_flag);
        if (ok)
          ok = mbar_wait(bar((first ? B_DOFULL : B_QFULL) + x % kRing), (x / kRing) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        if (first) {   // dV += P'^T dO_x
          mma_tm64(tmem + kColAcc0, tmem + kColS + 64u * (x & 1), ring1(x), x > 0);
          mma_commit(bar(B_DOEMPTY + x % kRing));
          mma_commit(bar(B_DVDONE + (x & 1)));
        } else {       // dK += dS'^T Q_x
          mma_tm64(tmem + kColAcc1, tmem + kColDA + 64u * (x & 1), ring0(x), x > 0);
          mma_commit(bar(B_QEMPTY + x % kRing));
          mma_commit(bar(B_DKDONE + (x & 1)));
        }
      }
      if (!ok) {
        set_status(a.status, kStatusTimeout);
        *abort_flag = 1;
      }
      mma_commit(bar(B_OUT));
    }
  } else if (warp < kWarpB) {
    // ---------------------------------------------------------- epilogue
    // Group g = (warp - 2) / 8 takes the sub-tiles x = g, g + 2, ...; warp w
    // owns TMEM lane quarter q4 = w % 4 (key rows 32 q4..) and the 32 query
    // columns 32 c2.. of the 64-column sub-tile.
    const int ew = warp - 2, g = ew >> 3, q4 = warp & 3, c2 = (ew >> 2) & 1;
    const int r = 32 * q4 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q4) << 16;
    const int j_loc = 128 * n + r;                  // this thread's key (row of S^T)
    const bool row_ok = j_loc < n_b;
    const int t_row = s + (row_ok ? j_loc : 0);
    const float nrm = a.norm_len > 0 ? static_cast<float>(a.norm_len) : static_cast<float>(n_b);
    const float inv_n = 1.0f / nrm;
    const int Lw = 2 * a.L - 1;
    // Key rows past the sequence end take the last token's timestamp, which
    // keeps their chunk plans on the cheap path (their elements are masked).
    const long long my_ts =
        TIME ? a.timestamps[checked(a.status, row_ok ? t_row : s + n_b - 1, a.T, BS_BWD_TS)] : 0;
    Stage* stg = reinterpret_cast<Stage*>(smem + kOffStage) + ew;
    float pw0 = 0.f, pw1 = 0.f;
    long long pt = 0;
    uint32_t pw = 0, plan_w = 0;                    // time plan word: prefetched, current
    // Staged for sub-tile x: the 63 position-bias diagonals of this warp's
    // 32 x 32 block (i - j = 128 (m - n) + 64 u + 32 c2 + cl - 32 q4 - lane,
    // index cl - lane + 31), its 32 query timestamps and this row's plan.
    auto prefetch = [&](int x) {
      const int cbase = 128 * (x >> 1) + 64 * (x & 1) + 32 * c2;   // query - 128 n
      if (POS) {
        const int t0 = cbase - 32 * q4 - 31 + lane + a.L - 1;
        const float* tab = a.rab_pos + static_cast<size_t>(h) * Lw;
        pw0 = (t0 >= 0 && t0 < Lw) ? __ldg(tab + t0) : 0.f;
        pw1 = (lane < 31 && t0 + 32 >= 0 && t0 + 32 < Lw) ? __ldg(tab + t0 + 32) : 0.f;
      }
      if (TIME) {
        const int i = 128 * n + cbase + lane;
        pt = a.timestamps[checked(a.status, s + (i < n_b ? i : n_b - 1), a.T, BS_BWD_TS)];
        // this row's plan against the block (rows past the end read the last row's)
        pw = a.plan_up[static_cast<size_t>(4 * n + (cbase >> 5)) * a.T +
                       checked(a.status, row_ok ? t_row : s + n_b - 1, a.T, BS_BWD_TS)];
      }
    };
    auto stage = [&]() {
      if (POS) {
        const float w0 = 0.5f * pw0, w1 = 0.5f * pw1;
        stg->w[lane] = w0;
        stg->w[32 + lane] = w1;
        // pairs (w[k], w[k+1]): k = lane and k = 32 + lane
        const float n0 = __shfl_down_sync(0xffffffffu, w0, 1);
        const float n1 = __shfl_down_sync(0xffffffffu, w1, 1);
        const float w32 = __shfl_sync(0xffffffffu, w1, 0);
        stg->wpk[lane] = pack_bf16x2(w0, lane < 31 ? n0 : w32);
        stg->wpk[32 + lane] = pack_bf16x2(w1, lane < 31 ? n1 : 0.f);
      }
      if (TIME) {
        stage_time(stg, lane, pt);
        plan_w = pw;
      }
      __syncwarp();
    };
    prefetch(g);
    stage();
    bool ok = true;
    for (int x = g; x < nx; x += 2) {
      const int u = x & 1, k = x >> 1, m = n + k;
      if (x + 2 < nx) prefetch(x + 2);
      const int c0 = 64 * u + 32 * c2;              // query column within tile m
      const bool diag = (m == n);
      const int qlim = n_b - 128 * m;               // valid query columns c < qlim
      // A block whose queries all precede its keys, or lie past the end, is
      // all zeros: the masked packed path without a time plan.  The plan
      // needs only the staged timestamps: taking it before the wait for S^T
      // and dA^T hides its chain of shared-memory loads there.
      const bool dead = (diag && c0 + 31 < 32 * q4) || c0 >= qlim;
      TimePlan tp{};
      int tb = TB_NONE;
      if (TIME && !dead) {
        tb = plan_unword(tp, plan_w);
        plan_values<true>(tp, tb, tt);
      }
      if (ok) ok = mbar_wait(bar(B_SFULL + u), k & 1, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      const uint32_t s_addr = tmem + lane_addr + kColS + 64u * u;
      const uint32_t a_addr = tmem + lane_addr + kColDA + 64u * u;
      uint32_t pk[16], dk[16];
      if (ok) {
        tc_fence_after();
        uint32_t sp[16], dp[16];
        load_pairs(s_addr + 32u * c2, sp);
        load_pairs(a_addr + 32u * c2, dp);
        {
          const bool msk = (diag && c0 < 32 * q4 + 31) || c0 + 31 >= qlim;
#define HSTU_DKV(TB_, M_)                                                                    \
  dkv_chunk<POS, TB_, M_>(sp, dp, stg, lane, r, c0, diag, qlim, tp, my_ts, tt, pk, dk)
          if (tb == TB_NONE) {
            if (msk) HSTU_DKV(TB_NONE, true); else HSTU_DKV(TB_NONE, false);
          } else if (tb == TB_CONST) {
            if (msk) HSTU_DKV(TB_CONST, true); else HSTU_DKV(TB_CONST, false);
          } else if (tb == TB_SPLIT) {
            if (msk) HSTU_DKV(TB_SPLIT, true); else HSTU_DKV(TB_SPLIT, false);
          } else if (tb == TB_MULTI) {
            HSTU_DKV(TB_MULTI, true);
          } else if (tb == TB_GEN32) {
            // the diagonal block and the one after it: buckets from the plan pass
            const int jd = 4 * n + q4, jc = 4 * m + (c0 >> 5);
            if (jc == jd || jc == jd + 1) {
              const uint4* src = a.near + static_cast<size_t>(row_ok ? t_row : s + n_b - 1) * 6 +
                                 (jc == jd ? 0 : 4);
              const uint4 b0 = __ldg(src), b1 = __ldg(src + 1);
              const uint32_t nbw[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
              dkv_chunk<POS, TB_BYTES, true>(sp, dp, stg, lane, r, c0, diag, qlim, tp, my_ts, tt,
                                             pk, dk, nbw);
            } else {
              HSTU_DKV(TB_GEN32, true);
            }
          } else {
            HSTU_DKV(TB_GEN64, true);
          }
#undef HSTU_DKV
        }
      }
      // P'^T and dS'^T go over this warp's own, already read S^T / dA^T
      // columns, so the warps of a group need not wait for one another.
      if (ok) {
        tmem_st16(s_addr + 32u * c2, pk);
        tmem_st16(a_addr + 32u * c2, dk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(B_PFULL + u));
      }
      if (x + 2 < nx) stage();
    }
    if (ok) ok = mbar_wait(bar(B_OUT), 0, abort_flag);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) {
      set_status(a.status, kStatusTimeout);
      *abort_flag = 1;
    }
    tc_fence_after();
    const int cq = ew >> 2;                         // 32-column quarter of dV, dK
    uint32_t vv[32], kv[32];
    tmem_ld32_nowait(tmem + lane_addr + kColAcc0 + 32u * cq, vv);
    tmem_ld32_nowait(tmem + lane_addr + kColAcc1 + 32u * cq, kv);
    tmem_wait_ld_dep(vv);
    tmem_wait_ld_dep(kv);
    if (ok && row_ok) {
      const size_t off = (static_cast<size_t>(checked(a.status, t_row, a.T, BS_BWD_ROW)) * a.H + h) * 128 + 32 * cq;
      uint4* dvp = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.dv) + off);
      uint4* dkp = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.dk) + off);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float* f = reinterpret_cast<const float*>(vv) + 8 * i;
        dvp[i] = make_uint4(pack_bf16x2(f[0] * inv_n, f[1] * inv_n), pack_bf16x2(f[2] * inv_n, f[3] * inv_n),
                            pack_bf16x2(f[4] * inv_n, f[5] * inv_n), pack_bf16x2(f[6] * inv_n, f[7] * inv_n));
        const float* e = reinterpret_cast<const float*>(kv) + 8 * i;
        dkp[i] = make_uint4(pack_bf16x2(e[0] * inv_n, e[1] * inv_n), pack_bf16x2(e[2] * inv_n, e[3] * inv_n),
                            pack_bf16x2(e[4] * inv_n, e[5] * inv_n), pack_bf16x2(e[6] * inv_n, e[7] * inv_n));
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if (lane == 0) mbar_wait(bar(B_OUT), 0, nullptr);
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}
}  // namespace dkv

// ===================================================================== dQ
namespace dq {
// smem: Q (T0), dO (T1), K sub-tiles (R0), V sub-tiles (R1)
enum {
  B_QDOFULL = 0,
  B_KFULL = 1,       // + ring slot
  B_KEMPTY = 4,      // + ring slot (count 2: S and dQ read K)
  B_VFULL = 7,
  B_VEMPTY = 10,
  B_SFULL = 13,      // + buffer (count 2: S and dA)
  B_SFREE = 15,      // + buffer (count kGroup): S read, its columns are free
  B_DSFULL = 17,     // + buffer (count kGroup): dS' written over dA
  B_DQDONE = 19,     // + buffer: dQ read dS', the dA columns are free
  B_OUT = 21         // count 3: every MMA of the three issuers done
};

template <bool POS, bool TIME>
__global__ void __launch_bounds__(kThreads, 1)
    hstu_bwd_dq_sm100(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_do,
                      const __grid_constant__ BwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = static_cast<int>(blockIdx.x % static_cast<unsigned>(a.H));
  const int idx = static_cast<int>(blockIdx.x / static_cast<unsigned>(a.H));
  const int m = a.max_tiles - 1 - idx / a.B;  // query tile, longest first
  const int b = idx % a.B;
  const int s = __ldg(a.offsets + b);
  const int e_ = __ldg(a.offsets + b + 1);
  int n_b = e_ - s;
  if (s < 0 || n_b < 0 || e_ > a.T || n_b > a.max_seq_len || (POS && n_b > a.L)) {
    if (threadIdx.x == 0 && h == 0 && m == 0) set_status(a.status, kStatusBadOffsets);
    n_b = 0;
  }
  if (128 * m >= n_b) return;
  const int nx = 2 * (m + 1);                 // key sub-tiles of tiles 0 .. m

  auto bar = [&](int i) { return sbase + kOffBar + 8u * i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  float* s_win = reinterpret_cast<float*>(smem + kOffWin);
  float* s_dt = reinterpret_cast<float*>(smem + kOffDT);

  if (threadIdx.x == 0) {
    for (int i = 0; i <= B_OUT; ++i) {
      uint32_t count = 1;
      if ((i >= B_KEMPTY && i < B_KEMPTY + kRing) || i == B_SFULL || i == B_SFULL + 1) count = 2;
      if (i == B_SFREE || i == B_SFREE + 1 || i == B_DSFULL || i == B_DSFULL + 1) count = kGroup;
      if (i == B_OUT) count = 3;
      mbar_init(bar(i), count);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sbase + kOffMisc, kTmemCols);
    tmem_relinquish();
  }
  if (warp >= 2 && warp < kWarpB) {
    const int et = threadIdx.x - 64;
    if (POS) {
      s_win[et] = 0.f;                        // 4 x 256 windows
      s_win[et + kEpi] = 0.f;
    }
    if (TIME && et < 128) s_dt[et] = 0.f;
  }
  TimeTables tt{};
  if (TIME) tt = init_tables(a, h, (warp >= 2 && warp < kWarpB) ? threadIdx.x - 64 : -1, smem);
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      const int qrow = checked(a.status, s + 128 * m, a.T, BS_BWD_TMA_Q);
      mbar_arrive_expect_tx(bar(B_QDOFULL), 2 * kTile);
      tma_load_3d(sbase + kOffT0, &tm_q, bar(B_QDOFULL), 0, h, qrow);
      tma_load_3d(sbase + kOffT0 + kHalf, &tm_q, bar(B_QDOFULL), 64, h, qrow);
      tma_load_3d(sbase + kOffT1, &tm_do, bar(B_QDOFULL), 0, h, qrow);
      tma_load_3d(sbase + kOffT1 + kHalf, &tm_do, bar(B_QDOFULL), 64, h, qrow);
      int k_last[kRing] = {-1, -1, -1}, v_last[kRing] = {-1, -1, -1};
      bool ok = true;
      for (int x = 0; x < nx && ok; ++x) {
        const int slot = x % kRing, use = x / kRing;
        const int krow = checked(a.status, s + 64 * x, a.T, BS_BWD_TMA_K);
        if (use > 0) ok = mbar_wait(bar(B_KEMPTY + slot), (use - 1) & 1, abort_flag);
        if (!ok) break;
        const uint32_t kd = sbase + kOffR0 + slot * kSubTile;
        mbar_arrive_expect_tx(bar(B_KFULL + slot), kSubTile);
        tma_load_3d(kd, &tm_k, bar(B_KFULL + slot), 0, h, krow);
        tma_load_3d(kd + kSub, &tm_k, bar(B_KFULL + slot), 64, h, krow);
        k_last[slot] = use;
        if (use > 0) ok = mbar_wait(bar(B_VEMPTY + slot), (use - 1) & 1, abort_flag);
        if (!ok) break;
        const uint32_t vd = sbase + kOffR1 + slot * kSubTile;
        mbar_arrive_expect_tx(bar(B_VFULL + slot), kSubTile);
        tma_load_3d(vd, &tm_v, bar(B_VFULL + slot), 0, h, krow);
        tma_load_3d(vd + kSub, &tm_v, bar(B_VFULL + slot), 64, h, krow);
        v_last[slot] = use;
      }
      if (!ok) {
        set_status(a.status, kStatusTimeout);
        *abort_flag = 1;
        mbar_wait(bar(B_QDOFULL), 0, nullptr);
        for (int sl = 0; sl < kRing; ++sl) {
          if (k_last[sl] >= 0) mbar_wait(bar(B_KFULL + sl), k_last[sl] & 1, nullptr);
          if (v_last[sl] >= 0) mbar_wait(bar(B_VFULL + sl), v_last[sl] & 1, nullptr);
        }
      }
    }
  } else if (warp == 1 || warp == kWarpB || warp == kWarpC) {
    // ---------------- MMA issuers: S (warp 1), dA (warp 18), dQ (warp 19)
    if (lane == 0) {
      bool ok = true;
      auto ring0 = [&](int x) { return sbase + kOffR0 + (x % kRing) * kSubTile; };
      auto ring1 = [&](int x) { return sbase + kOffR1 + (x % kRing) * kSubTile; };
      if (warp == 1 || warp == kWarpB) {
        const bool first = warp == 1;
        ok = mbar_wait(bar(B_QDOFULL), 0, abort_flag);
        for (int x = 0; x < nx && ok; ++x) {
          const int slot = x % kRing;
          ok = mbar_wait(bar((first ? B_KFULL : B_VFULL) + slot), (x / kRing) & 1, abort_flag);
          // buffer x % 2 was last used by sub-tile x - 2: S read by the
          // epilogue, dA (holding dS') read by the dQ MMA
          if (ok && x >= 2)
            ok = mbar_wait(bar((first ? B_SFREE : B_DQDONE) + (x & 1)), ((x - 2) >> 1) & 1,
                           abort_flag);
          if (!ok) break;
          tc_fence_after();
          if (first) {
            mma_n64(tmem + kColS + 64u * (x & 1), sbase + kOffT0, ring0(x));   // S = Q K_x^T
            mma_commit(bar(B_KEMPTY + slot));
          } else {
            mma_n64(tmem + kColDA + 64u * (x & 1), sbase + kOffT1, ring1(x));  // dA = dO V_x^T
            mma_commit(bar(B_VEMPTY + slot));
          }
          mma_commit(bar(B_SFULL + (x & 1)));
        }
      } else {
        for (int x = 0; x < nx && ok; ++x) {   // dQ += dS'_x K_x
          ok = mbar_wait(bar(B_DSFULL + (x & 1)), (x >> 1) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          mma_tm64(tmem + kColAcc0, tmem + kColDA + 64u * (x & 1), ring0(x), x > 0);
          mma_commit(bar(B_KEMPTY + x % kRing));
          mma_commit(bar(B_DQDONE + (x & 1)));
        }
      }
      if (!ok) {
        set_status(a.status, kStatusTimeout);
        *abort_flag = 1;
      }
      mma_commit(bar(B_OUT));
    }
  } else if (warp < kWarpB) {
    // ---------------------------------------------------------- epilogue
    // Group g takes the key sub-tiles x = g, g + 2, ...; warp w owns TMEM lane
    // quarter q4 (query rows 32 q4..) and the 32 key columns 32 c2.. of the
    // 64-column sub-tile.
    const int ew = warp - 2, g = ew >> 3, q4 = warp & 3, c2 = (ew >> 2) & 1;
    const int r = 32 * q4 + lane, et = threadIdx.x - 64, eg = et & (kGroup - 1);
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q4) << 16;
    const int i_loc = 128 * m + r;
    const bool row_ok = i_loc < n_b;
    const int t_row = s + (row_ok ? i_loc : 0);
    const float nrm = a.norm_len > 0 ? static_cast<float>(a.norm_len) : static_cast<float>(n_b);
    const float inv_n = 1.0f / nrm;
    const int Lw = 2 * a.L - 1;
    // Query rows past the sequence end (never stored) take the last token's
    // timestamp, which keeps their chunk plans on the cheap path.
    const long long my_ts =
        TIME ? a.timestamps[checked(a.status, row_ok ? t_row : s + n_b - 1, a.T, BS_BWD_TS)] : 0;
    Stage* stg = reinterpret_cast<Stage*>(smem + kOffStage) + ew;
    float pw0 = 0.f, pw1 = 0.f;
    long long pt = 0;
    uint32_t pw = 0, plan_w = 0;                    // time plan word: prefetched, current
    // Staged for sub-tile x: the 63 diagonals of this warp's 32 x 32 block
    // (i - j = 128 m + 32 q4 + lane - (64 x + 32 c2 + cl), index
    // lane - cl + 31), its 32 key timestamps and this row's plan.
    auto prefetch = [&](int x) {
      const int kbase = 64 * x + 32 * c2;          // first key of the warp's columns
      if (POS) {
        const int t0 = 128 * m + 32 * q4 - kbase - 31 + lane + a.L - 1;
        const float* tab = a.rab_pos + static_cast<size_t>(h) * Lw;
        pw0 = (t0 >= 0 && t0 < Lw) ? __ldg(tab + t0) : 0.f;
        pw1 = (lane < 31 && t0 + 32 >= 0 && t0 + 32 < Lw) ? __ldg(tab + t0 + 32) : 0.f;
      }
      if (TIME) {
        const int j = kbase + lane;
        pt = a.timestamps[checked(a.status, s + (j < n_b ? j : n_b - 1), a.T, BS_BWD_TS)];
        // this row's plan against the block (rows past the end read the last row's)
        pw = a.plan_dn[static_cast<size_t>(kbase >> 5) * a.T +
                       checked(a.status, row_ok ? t_row : s + n_b - 1, a.T, BS_BWD_TS)];
      }
    };
    auto stage = [&]() {
      if (POS) {
        const float w0 = 0.5f * pw0, w1 = 0.5f * pw1;
        stg->w[lane] = w0;
        stg->w[32 + lane] = w1;
        // pairs (w[k], w[k-1]): k = lane and k = 32 + lane
        const float p0 = __shfl_up_sync(0xffffffffu, w0, 1);
        const float p1 = __shfl_up_sync(0xffffffffu, w1, 1);
        const float w31 = __shfl_sync(0xffffffffu, w0, 31);
        stg->wpk[lane] = pack_bf16x2(w0, lane > 0 ? p0 : 0.f);
        stg->wpk[32 + lane] = pack_bf16x2(w1, lane > 0 ? p1 : w31);
      }
      if (TIME) {
        stage_time(stg, lane, pt);
        plan_w = pw;
      }
      __syncwarp();
    };
    prefetch(g);
    stage();
    bool ok = true;
    int run_k = -1;           // this row's running time-bucket sum of dS'
    float run_s = 0.f;
    // Window w of the group's sub-tile x holds the diagonal sums of
    // i - j = 128 (m - k) + w - 127 (k = x / 2); thread eg of the group moves
    // entry eg to d_rab_pos and clears it once every warp has added its part
    // (the group's sub-tile x + 2 adds to the other window, x + 4 to this one
    // again only after every warp has passed the start of x + 2).
    auto flush_window = [&](int x, bool ok_in) -> bool {
      bool okw = ok_in;
      if (okw) okw = mbar_wait(bar(B_DSFULL + (x & 1)), (x >> 1) & 1, abort_flag);
      okw = __all_sync(0xffffffffu, okw);
      const int k = x >> 1;
      float* w = s_win + 512 * g + 256 * (k & 1);
      if (okw && eg < 255) {
        const float v = w[eg];
        const int tbl = 128 * (m - k) + eg - 127 + a.L - 1;
        if (v != 0.f && tbl >= 0 && tbl < Lw)
          atomicAdd(a.d_rab_pos + static_cast<size_t>(h) * Lw + tbl, v * inv_n);
        w[eg] = 0.f;
      }
      return okw;
    };
    for (int x = g; x < nx; x += 2) {
      const int u = x & 1, k = x >> 1;              // k = key tile
      float* win = s_win + 512 * g + 256 * (k & 1);
      if (x + 2 < nx) prefetch(x + 2);
      // Sub-tile x - 2's diagonal sums are complete once its dS' phase is
      // (every warp adds them before arriving there), and so are the clears
      // of this sub-tile's window, made at the start of x - 2.
      if (POS && x >= 2) ok = flush_window(x - 2, ok);
      const int c0 = 64 * u + 32 * c2;              // key column within tile k
      const bool diag = (k == m);
      const int klim = n_b - 128 * k;               // valid key columns c < klim
      // A block whose keys all follow its queries, or lie past the end, or
      // whose rows all do, is all zeros: the masked packed path without a
      // time plan.  The plan needs only the staged timestamps: taking it
      // before the wait for S and dA hides its chain of shared-memory loads.
      const bool dead =
          (diag && c0 > 32 * q4 + 31) || c0 >= klim || !__any_sync(0xffffffffu, row_ok);
      TimePlan tp{};
      int tb = TB_NONE;
      if (TIME && !dead) {
        tb = plan_unword(tp, plan_w);
        plan_values<false>(tp, tb, tt);
      }
      if (ok) ok = mbar_wait(bar(B_SFULL + u), k & 1, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      const uint32_t s_addr = tmem + lane_addr + kColS + 64u * u;
      const uint32_t a_addr = tmem + lane_addr + kColDA + 64u * u;
      uint32_t dk[16];
      if (ok) {
        tc_fence_after();
        uint32_t sp[16], dp[16];
        load_pairs(s_addr + 32u * c2, sp);
        tc_fence_before();
        mbar_arrive(bar(B_SFREE + u));            // S read: its buffer may take S of x + 2
        load_pairs(a_addr + 32u * c2, dp);
        {
          // window index r - c + 127 of the block's diagonals
          const int wbase = 32 * q4 - c0 + 127;
          const bool msk = (diag && c0 + 31 > 32 * q4) || c0 + 31 >= klim ||
                           !__all_sync(0xffffffffu, row_ok);
#define HSTU_DQ(TB_, M_)                                                                    \
  dq_chunk<POS, TB_, M_>(sp, dp, stg, lane, r, c0, diag, klim, row_ok, tp, my_ts, tt, win, \
                         wbase, s_dt, dk, run_k, run_s)
          if (tb == TB_NONE) {
            if (msk) HSTU_DQ(TB_NONE, true); else HSTU_DQ(TB_NONE, false);
          } else if (tb == TB_CONST) {
            if (msk) HSTU_DQ(TB_CONST, true); else HSTU_DQ(TB_CONST, false);
          } else if (tb == TB_SPLIT) {
            if (msk) HSTU_DQ(TB_SPLIT, true); else HSTU_DQ(TB_SPLIT, false);
          } else if (tb == TB_MULTI) {
            HSTU_DQ(TB_MULTI, true);
          } else if (tb == TB_GEN32) {
            // the diagonal block and the one before it: buckets from the plan pass
            const int jd = 4 * m + q4, jc = 4 * k + (c0 >> 5);
            if (jc == jd || jc == jd - 1) {
              const uint4* src = a.near + static_cast<size_t>(row_ok ? t_row : s + n_b - 1) * 6 +
                                 (jc == jd ? 0 : 2);
              const uint4 b0 = __ldg(src), b1 = __ldg(src + 1);
              const uint32_t nbw[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
              dq_chunk<POS, TB_BYTES, true>(sp, dp, stg, lane, r, c0, diag, klim, row_ok, tp, my_ts,
                                            tt, win, wbase, s_dt, dk, run_k, run_s, nbw);
            } else {
              HSTU_DQ(TB_GEN32, true);
            }
          } else {
            HSTU_DQ(TB_GEN64, true);
          }
#undef HSTU_DQ
        }
      }
      // dS' goes over this warp's own, already read dA columns, so the warps
      // of a group need not wait for one another.
      if (ok) {
        tmem_st16(a_addr + 32u * c2, dk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(B_DSFULL + u));
      }
      if (x + 2 < nx) stage();
    }
    // the group's last sub-tile
    const int x_last = g + 2 * ((nx - 1 - g) >> 1);
    if (POS && x_last >= 0 && x_last < nx) ok = flush_window(x_last, ok);
    // dQ = (1/N) sum dS' K
    if (ok) ok = mbar_wait(bar(B_OUT), 0, abort_flag);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) {
      set_status(a.status, kStatusTimeout);
      *abort_flag = 1;
    }
    tc_fence_after();
    const int cq = ew >> 2;
    uint32_t qv[32];
    tmem_ld32_nowait(tmem + lane_addr + kColAcc0 + 32u * cq, qv);
    tmem_wait_ld_dep(qv);
    if (ok && row_ok) {
      uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.dq) +
                                            (static_cast<size_t>(t_row) * a.H + h) * 128 + 32 * cq);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float* f = reinterpret_cast<const float*>(qv) + 8 * i;
        dst[i] = make_uint4(pack_bf16x2(f[0] * inv_n, f[1] * inv_n), pack_bf16x2(f[2] * inv_n, f[3] * inv_n),
                            pack_bf16x2(f[4] * inv_n, f[5] * inv_n), pack_bf16x2(f[6] * inv_n, f[7] * inv_n));
      }
    }
    if (TIME) {
      if (run_k >= 0) atomicAdd(&s_dt[run_k], run_s);
      named_bar_sync(3, kEpi);
      if (et < a.nb && s_dt[et] != 0.f)
        atomicAdd(a.d_rab_time + static_cast<size_t>(h) * a.nb + et, s_dt[et] * inv_n);
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if (lane == 0) mbar_wait(bar(B_OUT), 0, nullptr);
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}
}  // namespace dq

// `configured` caches, per device, that the kernel's shared-memory opt-in has
// been set; concurrent host threads at worst set the same attribute twice.
template <typename K>
cudaError_t launch_plain(K kernel, unsigned grid, const CUtensorMap* maps, const BwdArgs& a,
                         cudaStream_t stream, std::atomic<bool>* configured) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  const bool cached = dev >= 0 && dev < 64;
  if (!cached || !configured[dev].load(std::memory_order_acquire)) {
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (err != cudaSuccess) return err;
    if (cached) configured[dev].store(true, std::memory_order_release);
  }
  kernel<<<grid, kThreads, kSmem, stream>>>(maps[0], maps[1], maps[2], maps[3], a);
  return cudaGetLastError();
}

template <bool POS, bool TIME>
cudaError_t launch_variant(const BwdArgs& a, const CUtensorMap* maps, cudaStream_t stream) {
  static std::atomic<bool> conf_dq[64], conf_dkv[64];   // zero-initialised: false
  const unsigned grid = static_cast<unsigned>(a.H) * static_cast<unsigned>(a.B) *
                        static_cast<unsigned>(a.max_tiles);
  // maps: q, k, v, dO with 128-row boxes, then with 64-row boxes
  const CUtensorMap mq[4] = {maps[0], maps[5], maps[6], maps[3]};   // Q, dO resident; K, V rings
  const CUtensorMap mk[4] = {maps[4], maps[1], maps[2], maps[7]};   // K, V resident; Q, dO rings
  cudaError_t err = launch_plain(dq::hstu_bwd_dq_sm100<POS, TIME>, grid, mq, a, stream, conf_dq);
  if (err != cudaSuccess) return err;
  return launch_plain(dkv::hstu_bwd_dkdv_sm100<POS, TIME>, grid, mk, a, stream, conf_dkv);
}

}  // namespace

// maps: q, k, v, dO ([T, H, 128] bf16) with 128-row boxes (0..3), then with
// 64-row boxes (4..7).  The LN/gate part (dO, dU) must already be in a.dO /
// a.du.
cudaError_t launch_bwd_attn_bf16_sm100(const BwdArgs& a, const CUtensorMap* maps,
                                       cudaStream_t stream) {
  if (a.B == 0 || a.max_tiles == 0) return cudaSuccess;
  const bool pos = a.rab_pos != nullptr, tim = a.rab_time != nullptr;
  if (tim) {
    if (!a.plan_dn || !a.plan_up || a.plan_j < 4 * a.max_tiles) return cudaErrorInvalidValue;
    PlanArgs pa{};
    pa.offsets = a.offsets;
    pa.timestamps = a.timestamps;
    pa.plan_dn = a.plan_dn;
    pa.plan_up = a.plan_up;
    pa.near = a.near;
    pa.status = a.status;
    pa.B = a.B;
    pa.T = a.T;
    pa.max_seq_len = a.max_seq_len;
    pa.max_tiles = a.max_tiles;
    pa.plan_j = a.plan_j;
    pa.bt = a.bt;
    const cudaError_t err = launch_time_plans(pa, stream);
    if (err != cudaSuccess) return err;
  }
  if (pos && tim) return launch_variant<true, true>(a, maps, stream);
  if (pos) return launch_variant<true, false>(a, maps, stream);
  if (tim) return launch_variant<false, true>(a, maps, stream);
  return launch_variant<false, false>(a, maps, stream);
}

}  // namespace hstu
