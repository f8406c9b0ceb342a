// cand_sm100.cu -- candidate scoring against cached histories (M-FALCON) on
// sm_100a.
//
// "HSTU Hierarchical Sequential Transduction Units", §6 Why it works, names
// M-FALCON: micro-batched candidate scoring that reuses the history's keys
// and values.  Candidate c of user b is scored as the token that follows the
// user's n_b history tokens, on its own: it attends to every history token
// j < n_b (relative position n_b - j, time bucket of t_c - t_j) and to itself
// (relative position 0, time difference 0), never to another candidate, and
// is normalised by norm_len or n_b + 1.  Its output row is therefore the last
// row of the causal forward over (history, c).
//
// One CTA per (user, micro-batch of 128 candidates, head): every history key
// and value tile is brought in once by TMA and serves the whole micro-batch.
//   warp 0       TMA: the micro-batch's Q tile, then K and V tiles (2 stages)
//   warp 1       TMEM allocation; S = Q K^T into one of two S buffers, and
//                O += P V with P read from TMEM
//   warps 2..17  epilogue: warp w owns TMEM lane quarter w % 4 and the 32 S
//                columns 32 ((w-2)/4) ..; bias + SiLU + key mask, P (bf16)
//                written over its own S columns; then O plus the self term,
//                times 1/N, staged in fp32 for the LayerNorm over heads, which
//                the last of the H head CTAs of the micro-batch applies.
// Every wait is bounded; a wait that runs out sets the timeout bit of the
// status word and the CTA leaves through the same barriers.
#include <cuda_bf16.h>

#include <atomic>

#include "bounds.cuh"
#include "internal.h"
#include "ptx.cuh"
#include "tile_math.cuh"

namespace hstu {
namespace {

constexpr int kThreads = 576;
constexpr int kEpiWarps = 16;
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kHalf = 16384;               // 128 rows x 64 bf16
constexpr int kTile = 2 * kHalf;           // 128 x 128 bf16
constexpr int kStages = 2;
constexpr int kColO = 256;                 // O accumulator: TMEM columns 256..383
constexpr int kTmemCols = 512;

constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kTile;
constexpr int kOffV = kOffK + kStages * kTile;
constexpr int kOffBar = kOffV + kStages * kTile;
enum {
  B_QFULL = 0,
  B_KFULL = 1,     // + stage
  B_KEMPTY = 3,
  B_VFULL = 5,
  B_VEMPTY = 7,
  B_SFULL = 9,     // + S buffer
  B_PFULL = 11,
  B_PVDONE = 13,
  B_OFULL = 15,
  kNumBars = 16
};
constexpr int kOffMisc = kOffBar + kNumBars * 8;   // [0] TMEM base, [1] abort, [2] last-arriver
constexpr int kOffThr = kOffMisc + 16;             // long long [kThrLen]
constexpr int kOffFirst = kOffThr + kThrLen * 8;   // signed char [64]
constexpr int kOffRabT = kOffFirst + 64;           // float [kMaxBuckets]: this head's time bias
constexpr int kOffPart = kOffRabT + kMaxBuckets * 4;   // float [4][128] LayerNorm partials
constexpr int kOffRabH = kOffPart + 4 * 128 * 4;       // float [kMaxBuckets]: half time bias
constexpr int kOffOct = kOffRabH + kMaxBuckets * 4;    // uint4 [32]: per-octave thresholds
constexpr int kOffThr32 = kOffOct + 32 * 16;           // unsigned [kMaxBuckets]
constexpr int kOffStage = kOffThr32 + kMaxBuckets * 4; // per epilogue warp: Stage
// Per epilogue warp, the chunk's 32 keys: half position-bias pairs of
// neighbouring columns and the keys' timestamps (low 32 bits).
struct Stage {
  uint32_t ppk[16];
  uint32_t ts32[32];
};
constexpr int kSmem = kOffStage + kEpiWarps * static_cast<int>(sizeof(Stage)) + 1024;
static_assert(kOffOct % 16 == 0 && kOffStage % 16 == 0, "table alignment");
static_assert(kSmem <= 227 * 1024, "shared memory per CTA");

// The bucket tables of the epilogue in shared memory (half time bias).
struct CandTab {
  const uint4* oct_;
  const unsigned* thr32_;
  const float* rabh_;
  __device__ __forceinline__ const uint4* oct() const { return oct_; }
  __device__ __forceinline__ const unsigned* thr32() const { return thr32_; }
  __device__ __forceinline__ const float* rabt() const { return rabh_; }
};

constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, false, true);

__device__ __forceinline__ bool checked(bool ok, int* status) {
  if (!ok && status) atomicOr(status, kStatusTimeout);
  return ok;
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// SiLU(x) = x/2 (1 + tanh(x/2))
__device__ __forceinline__ float silu_t(float x) {
  const float hx = 0.5f * x;
  return fmaf(hx, tanh_approx(hx), hx);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

}  // namespace

// P pairs of one 32-key chunk on bf16 pairs: half bias (position pair from
// the staging, time pair from the plan or per element) added to S/2, SiLU as
// hx (1 + tanh hx), keys at or past nvalid set to exactly 0.
template <bool POS, int TB>
__device__ __forceinline__ void cand_pairs(const uint32_t (&sv)[32], const Stage* stg,
                                           const TimePlan& tp, uint32_t my32, const CandTab& tab,
                                           int nvalid, uint32_t (&packed)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    uint32_t hb = POS ? stg->ppk[i] : 0u;
    if (TB == TB_GEN32) {
      const int2 kb = gen_bucket_pair(stg->ts32, i, my32, tab);
      const uint32_t t2 = pack_bf16x2(tab.rabt()[kb.x], tab.rabt()[kb.y]);
      hb = POS ? hadd2(hb, t2) : t2;
    } else if (TB != TB_NONE) {
      hb = POS ? hadd2(hb, plan_pair<TB>(tp, i)) : plan_pair<TB>(tp, i);
    }
    const uint32_t s2 = pack_bf16x2(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1]));
    const uint32_t hx = hfma2(s2, kHalfPair, hb);
    const uint32_t keep = (2 * i < nvalid ? 0x0000FFFFu : 0u) | (2 * i + 1 < nvalid ? 0xFFFF0000u : 0u);
    packed[i] = hfma2(hx, tanh2(hx), hx) & keep;
  }
}

template <bool POS, bool TIME>
__global__ void __launch_bounds__(kThreads, 1)
    hstu_cand_sm100(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CandArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto bar = [&](int i) { return sbase + kOffBar + 8u * i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  long long* s_thr = reinterpret_cast<long long*>(smem + kOffThr);
  signed char* s_first = reinterpret_cast<signed char*>(smem + kOffFirst);
  float* s_rabt = reinterpret_cast<float*>(smem + kOffRabT);
  float* s_part = reinterpret_cast<float*>(smem + kOffPart);

  // CTA (head, rank, micro-batch), the micro-batch fastest: the micro-batches
  // of one (user, head) run together and share its history tiles in L2, and
  // within each head the user with the longest history comes first
  const unsigned bb = static_cast<unsigned>(a.B), tt_ = static_cast<unsigned>(a.max_tiles);
  const int mt = static_cast<int>(blockIdx.x % tt_);
  const int rank = static_cast<int>((blockIdx.x / tt_) % bb);
  const int h = static_cast<int>(blockIdx.x / tt_ / bb);
  const int b = a.order ? __ldg(a.order + rank) : rank;
  const int c0 = __ldg(a.cand_offsets + b);
  const int cb = __ldg(a.cand_offsets + b + 1) - c0;
  const int s = __ldg(a.offsets + b);
  const int nb = __ldg(a.offsets + b + 1) - s;
  // Offsets that contradict the sizes: record and leave (uniform over the CTA).
  if (c0 < 0 || cb < 0 || c0 + cb > a.C || cb > 128 * a.max_tiles || s < 0 || nb < 0 ||
      s + nb > a.T || nb > a.max_seq_len || (POS && nb + 1 > a.L)) {
    if (threadIdx.x == 0 && mt == 0 && a.status) atomicOr(a.status, kStatusBadOffsets);
    return;
  }
  if (128 * mt >= cb) return;   // this micro-batch is past the user's candidates
  const int nt = (nb + 127) / 128;
  const int D = a.H * 128;

  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), 1);
    for (int st = 0; st < kStages; ++st) {
      mbar_init(bar(B_KFULL + st), 1);
      mbar_init(bar(B_KEMPTY + st), 1);
      mbar_init(bar(B_VFULL + st), 1);
      mbar_init(bar(B_VEMPTY + st), 1);
      mbar_init(bar(B_SFULL + st), 1);
      mbar_init(bar(B_PFULL + st), kEpiWarps);
      mbar_init(bar(B_PVDONE + st), 1);
    }
    mbar_init(bar(B_OFULL), 1);
    *abort_flag = 0;
    misc[2] = 0;
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < kThrLen; i += kThreads) s_thr[i] = a.bt.thr[i];
  for (int i = threadIdx.x; i < 64; i += kThreads) s_first[i] = a.bt.first_k[i];
  CandTab tab;
  tab.oct_ = reinterpret_cast<const uint4*>(smem + kOffOct);
  tab.thr32_ = reinterpret_cast<const unsigned*>(smem + kOffThr32);
  tab.rabh_ = reinterpret_cast<const float*>(smem + kOffRabH);
  if (TIME) {
    for (int i = threadIdx.x; i < a.nb; i += kThreads) {
      const float v = __ldg(a.rab_time + h * a.nb + i);
      s_rabt[i] = v;
      reinterpret_cast<float*>(smem + kOffRabH)[i] = 0.5f * v;
    }
    for (int i = threadIdx.x; i < 32; i += kThreads)
      reinterpret_cast<uint4*>(smem + kOffOct)[i] = a.bt.oct[i];
    for (int i = threadIdx.x; i < kMaxBuckets; i += kThreads)
      reinterpret_cast<unsigned*>(smem + kOffThr32)[i] = a.bt.thr32[i];
  }
  if (warp == 1) {
    tmem_alloc(sbase + kOffMisc, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && nt > 0) {
      int klast[kStages] = {-1, -1}, vlast[kStages] = {-1, -1};
      bool ok = true;
      const int qrow = checked(a.status, c0 + 128 * mt, a.C, BS_CAND_TMA);
      mbar_arrive_expect_tx(bar(B_QFULL), kTile);
      tma_load_3d(sbase + kOffQ, &tm_q, bar(B_QFULL), 0, h, qrow);
      tma_load_3d(sbase + kOffQ + kHalf, &tm_q, bar(B_QFULL), 64, h, qrow);
      for (int n = 0; n < nt && ok; ++n) {
        const int st = n % kStages, use = n / kStages;
        if (use > 0)
          ok = checked(mbar_wait(bar(B_KEMPTY + st), (use - 1) & 1, abort_flag), a.status);
        if (!ok) break;
        const int krow = checked(a.status, s + 128 * n, a.T, BS_CAND_TMA);
        mbar_arrive_expect_tx(bar(B_KFULL + st), kTile);
        tma_load_3d(sbase + kOffK + st * kTile, &tm_k, bar(B_KFULL + st), 0, h, krow);
        tma_load_3d(sbase + kOffK + st * kTile + kHalf, &tm_k, bar(B_KFULL + st), 64, h, krow);
        klast[st] = use;
        if (use > 0)
          ok = checked(mbar_wait(bar(B_VEMPTY + st), (use - 1) & 1, abort_flag), a.status);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(B_VFULL + st), kTile);
        tma_load_3d(sbase + kOffV + st * kTile, &tm_v, bar(B_VFULL + st), 0, h, krow);
        tma_load_3d(sbase + kOffV + st * kTile + kHalf, &tm_v, bar(B_VFULL + st), 64, h, krow);
        vlast[st] = use;
      }
      if (!ok) {
        *abort_flag = 1;
        // the copies already issued land before shared memory is released
        mbar_wait(bar(B_QFULL), 0, nullptr);
        for (int st = 0; st < kStages; ++st) {
          if (klast[st] >= 0) mbar_wait(bar(B_KFULL + st), klast[st] & 1, nullptr);
          if (vlast[st] >= 0) mbar_wait(bar(B_VFULL + st), vlast[st] & 1, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      if (nt > 0) {
        ok = checked(mbar_wait(bar(B_QFULL), 0, abort_flag), a.status);
        auto issue_s = [&](int n) {
          const int st = n % kStages;
          bool r = checked(mbar_wait(bar(B_KFULL + st), (n / kStages) & 1, abort_flag), a.status);
          // S buffer st was last read (as P) by the P.V MMAs of tile n - 2
          if (r && n >= 2)
            r = checked(mbar_wait(bar(B_PVDONE + st), ((n - 2) / kStages) & 1, abort_flag),
                        a.status);
          if (!r) return false;
          tc_fence_after();
          const uint32_t qa = sbase + kOffQ, ka = sbase + kOffK + st * kTile;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t off = (ks >> 2) * kHalf + (ks & 3) * 32;
            mma_ss(tmem + 128u * st, sw128_desc(qa + off, 16, 1024),
                   sw128_desc(ka + off, 16, 1024), kIdescS, ks > 0 ? 1u : 0u);
          }
          mma_commit(bar(B_KEMPTY + st));
          mma_commit(bar(B_SFULL + st));
          return true;
        };
        if (ok) ok = issue_s(0);
        for (int n = 0; n < nt && ok; ++n) {
          if (n + 1 < nt) ok = issue_s(n + 1);
          const int st = n % kStages;
          if (ok)
            ok = checked(mbar_wait(bar(B_PFULL + st), (n / kStages) & 1, abort_flag), a.status);
          if (ok)
            ok = checked(mbar_wait(bar(B_VFULL + st), (n / kStages) & 1, abort_flag), a.status);
          if (!ok) break;
          tc_fence_after();
          const uint32_t va = sbase + kOffV + st * kTile;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            // keys 16ks..16ks+15: P of S column group ks/2 sits in its first 16 columns
            mma_ts(tmem + kColO, tmem + 128u * st + 32u * (ks >> 1) + 8u * (ks & 1),
                   sw128_desc(va + ks * 2048, kHalf, 1024), kIdescPV, (n > 0 || ks > 0) ? 1u : 0u);
          mma_commit(bar(B_VEMPTY + st));
          mma_commit(bar(B_PVDONE + st));
        }
      }
      if (!ok) *abort_flag = 1;
      mma_commit(bar(B_OFULL));
      // TMEM is released only after every MMA issued here has completed.
      mbar_wait(bar(B_OFULL), 0, nullptr);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2, q4 = warp & 3, cs = ew >> 2;
    const int r = 32 * q4 + lane;              // micro-batch row = TMEM lane
    const int i_loc = 128 * mt + r;
    const bool row_ok = i_loc < cb;
    const int cand = c0 + (row_ok ? i_loc : 0);
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(32 * q4) << 16);
    const long long my_ts = TIME ? __ldg(a.cand_ts + checked(a.status, cand, a.C, BS_CAND_ROW)) : 0ll;
    // rpos[d] = this head's position bias at relative position d >= 0
    const float* rpos = POS ? a.rab_pos + static_cast<size_t>(h) * (2 * a.L - 1) + (a.L - 1) : nullptr;
    Stage* stg = reinterpret_cast<Stage*>(smem + kOffStage) + ew;
    bool ok = true;
    for (int n = 0; n < nt; ++n) {
      const int st = n % kStages;
      // lane c stages column c of this warp's 32 keys; the row loop reads it by shuffle
      const int j = 128 * n + 32 * cs + lane;
      const bool jv = j < nb;
      const float pb = (POS && jv) ? __ldg(rpos + (nb - j)) : 0.f;
      const long long kts = (TIME && jv) ? __ldg(a.timestamps + checked(a.status, s + j, a.T, BS_CAND_TS)) : 0ll;
      // this candidate's time plan against the chunk (the plan pass)
      const uint32_t pw = (TIME && 128 * n + 32 * cs < nb)
                              ? __ldg(a.plan + static_cast<size_t>(4 * n + cs) * a.C + cand)
                              : 0u;
      if (ok) ok = checked(mbar_wait(bar(B_SFULL + st), (n / kStages) & 1, abort_flag), a.status);
      ok = __all_sync(0xffffffffu, ok);   // the TMEM accesses below are warp-collective
      if (!ok) break;
      tc_fence_after();
      const uint32_t saddr = lane_addr + 128u * st + 32u * cs;
      uint32_t sv[32];
      tmem_ld32_nowait(saddr, sv);
      tmem_wait_ld_dep(sv);
      const int nvalid = nb - (128 * n + 32 * cs);   // columns of this chunk that are history keys
      uint32_t packed[16];
      if (nvalid <= 0) {
        // past the history: every column is masked
#pragma unroll
        for (int i = 0; i < 16; ++i) packed[i] = 0u;
      } else {
        // Stage this warp's 32 keys: the half position-bias pair (pb_c, pb_c+1)
        // lane c = 2i forms, and the timestamps, keys past the history
        // repeating the last one (which keeps them ascending; they are masked).
        __syncwarp();
        if (POS) {
          const float hb = 0.5f * pb;
          const float nxt = __shfl_down_sync(0xffffffffu, hb, 1);
          if ((lane & 1) == 0) stg->ppk[lane >> 1] = pack_bf16x2(hb, nxt);
        }
        TimePlan tp{};
        int tb = TB_NONE;
        if (TIME) {
          // the keys' timestamps for the per-element paths (past the history:
          // the last one; those columns are masked)
          const long long last = __shfl_sync(0xffffffffu, kts, nvalid < 32 ? nvalid - 1 : 31);
          stg->ts32[lane] = static_cast<uint32_t>(jv ? kts : last);
          tb = plan_unword(tp, pw);
          plan_values<false>(tp, tb, tab);
        }
        __syncwarp();
        const uint32_t my32 = static_cast<uint32_t>(my_ts);
        if (tb == TB_GEN64) {
          // time spans of 2^31 or more: fp32 with the 64-bit bucket search
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float p2[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int c = 2 * i + e;
              float x = __uint_as_float(sv[c]);
              if (POS) x += __shfl_sync(0xffffffffu, pb, c);
              const long long kt = __shfl_sync(0xffffffffu, kts, c);
              x += s_rabt[time_bucket(my_ts - kt, s_thr, s_first)];
              p2[e] = c < nvalid ? silu_t(x) : 0.f;
            }
            packed[i] = pack2(p2[0], p2[1]);
          }
        } else {
#define HSTU_CAND(TB_) cand_pairs<POS, TB_>(sv, stg, tp, my32, tab, nvalid, packed)
          if (tb == TB_NONE) {
            HSTU_CAND(TB_NONE);
          } else if (tb == TB_CONST) {
            HSTU_CAND(TB_CONST);
          } else if (tb == TB_SPLIT) {
            HSTU_CAND(TB_SPLIT);
          } else if (tb == TB_MULTI) {
            HSTU_CAND(TB_MULTI);
          } else {
            HSTU_CAND(TB_GEN32);
          }
#undef HSTU_CAND
        }
      }
      tmem_st16(saddr, packed);   // over this warp's own S columns, already read
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_PFULL + st));
    }
    if (ok) ok = checked(mbar_wait(bar(B_OFULL), 0, abort_flag), a.status);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && lane == 0) *abort_flag = 1;

    // ---------------------------------- O of this head, plus the self term, / N
    float o[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) o[c] = 0.f;
    if (ok && nt > 0) {
      tc_fence_after();
      uint32_t ov[32];
      tmem_ld32_nowait(lane_addr + kColO + 32u * cs, ov);
      tmem_wait_ld_dep(ov);
#pragma unroll
      for (int c = 0; c < 32; ++c) o[c] = __uint_as_float(ov[c]);
    }
    {
      const size_t hrow = (static_cast<size_t>(cand) * a.H + h) * 128;
      const uint4* q4p = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q) + hrow);
      const uint4* k4p = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.k) + hrow);
      float dot = 0.f;
#pragma unroll 4
      for (int i = 0; i < 16; ++i) {
        const uint4 qa = __ldg(q4p + i), ka = __ldg(k4p + i);
        const uint32_t qw[4] = {qa.x, qa.y, qa.z, qa.w}, kw[4] = {ka.x, ka.y, ka.z, ka.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          dot = fmaf(bf16_lo(qw[e]), bf16_lo(kw[e]), dot);
          dot = fmaf(bf16_hi(qw[e]), bf16_hi(kw[e]), dot);
        }
      }
      float x = dot;
      if (POS) x += __ldg(rpos);
      if (TIME) x += s_rabt[time_bucket(0ll, s_thr, s_first)];
      const float aii = silu_t(x);
      const float inv_n = 1.0f / static_cast<float>(a.norm_len > 0 ? a.norm_len : nb + 1);
      const uint4* v4p = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.v) +
                                                        hrow + 32 * cs);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 va = __ldg(v4p + i);
        const uint32_t vw[4] = {va.x, va.y, va.z, va.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          o[8 * i + 2 * e] = (o[8 * i + 2 * e] + aii * bf16_lo(vw[e])) * inv_n;
          o[8 * i + 2 * e + 1] = (o[8 * i + 2 * e + 1] + aii * bf16_hi(vw[e])) * inv_n;
        }
      }
      if (row_ok) {
        float4* dst = reinterpret_cast<float4*>(a.o_ws + static_cast<size_t>(cand) * D + h * 128 + 32 * cs);
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
      }
    }

    // ---------------------------------- the last head CTA: LayerNorm over heads, gate
    __threadfence();
    named_bar_sync(1, kEpiThreads);
    if (ew == 0 && lane == 0) {
      unsigned* cnt = a.cnt + checked(a.status, static_cast<size_t>(b) * a.max_tiles + mt,
                                      static_cast<long long>(a.B) * a.max_tiles, BS_CAND_CNT);
      const unsigned old = atomicAdd(cnt, 1u);
      const bool last = old == static_cast<unsigned>(a.H - 1);
      if (last) *cnt = 0u;   // re-armed: every head of this micro-batch has counted
      misc[2] = last ? 1u : 0u;
    }
    named_bar_sync(1, kEpiThreads);
    if (*reinterpret_cast<volatile uint32_t*>(misc + 2)) {
      __threadfence();
      const int w4 = D / 4;                      // columns of the row this thread takes
      const float* orow = a.o_ws + static_cast<size_t>(cand) * D + cs * w4;
      float sum = 0.f;
      if (row_ok)
        for (int i = 0; i < w4; i += 4) {
          const float4 x = ld_global_cg_f4(orow + i);
          sum += (x.x + x.y) + (x.z + x.w);
        }
      s_part[cs * 128 + r] = sum;
      named_bar_sync(1, kEpiThreads);
      const float mean = (s_part[r] + s_part[128 + r] + s_part[256 + r] + s_part[384 + r]) /
                         static_cast<float>(D);
      named_bar_sync(1, kEpiThreads);
      float sq = 0.f;
      if (row_ok)
        for (int i = 0; i < w4; i += 4) {
          const float4 x = ld_global_cg_f4(orow + i);
          const float d0 = x.x - mean, d1 = x.y - mean, d2 = x.z - mean, d3 = x.w - mean;
          sq += (d0 * d0 + d1 * d1) + (d2 * d2 + d3 * d3);
        }
      s_part[cs * 128 + r] = sq;
      named_bar_sync(1, kEpiThreads);
      const float var = (s_part[r] + s_part[128 + r] + s_part[256 + r] + s_part[384 + r]) /
                        static_cast<float>(D);
      const float rstd = 1.0f / sqrtf(var + a.eps);
      if (row_ok) {
        const int col0 = cs * w4;
        const __nv_bfloat16* urow = static_cast<const __nv_bfloat16*>(a.u) +
                                    static_cast<size_t>(cand) * D + col0;
        __nv_bfloat16* yrow = static_cast<__nv_bfloat16*>(a.y) + static_cast<size_t>(cand) * D + col0;
        for (int i = 0; i < w4; i += 8) {
          const float4 x0 = ld_global_cg_f4(orow + i), x1 = ld_global_cg_f4(orow + i + 4);
          const float xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
          const uint4 uw = __ldg(reinterpret_cast<const uint4*>(urow + i));
          const uint32_t us[4] = {uw.x, uw.y, uw.z, uw.w};
          uint32_t yw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float yy[2];
#pragma unroll
            for (int f = 0; f < 2; ++f) {
              const int c = col0 + i + 2 * e + f;
              const float g = a.ln_weight ? __ldg(a.ln_weight + c) : 1.f;
              const float bb = a.ln_bias ? __ldg(a.ln_bias + c) : 0.f;
              const float uu = f ? bf16_hi(us[e]) : bf16_lo(us[e]);
              yy[f] = fmaf((xv[2 * e + f] - mean) * rstd, g, bb) * silu_t(uu);
            }
            yw[e] = pack2(yy[0], yy[1]);
          }
          *reinterpret_cast<uint4*>(yrow + i) = make_uint4(yw[0], yw[1], yw[2], yw[3]);
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <bool POS, bool TIME>
cudaError_t launch_t(const CandArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                     const CUtensorMap& tv, cudaStream_t stream) {
  static std::atomic<bool> configured[64];   // per device: shared-memory opt-in done
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64 || !configured[dev].load(std::memory_order_acquire)) {
    err = cudaFuncSetAttribute(hstu_cand_sm100<POS, TIME>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (err != cudaSuccess) return err;
    if (dev >= 0 && dev < 64) configured[dev].store(true, std::memory_order_release);
  }
  const dim3 grid(static_cast<unsigned>(a.B) * static_cast<unsigned>(a.max_tiles) *
                  static_cast<unsigned>(a.H));
  hstu_cand_sm100<POS, TIME><<<grid, kThreads, kSmem, stream>>>(tq, tk, tv, a);
  return cudaGetLastError();
}

// The users' ranks by history length (longest first, ties by index): each
// thread counts the users that come before its own, a few thousand at most.
__global__ void cand_order(const int32_t* offsets, int B, int* order) {
  const int b = static_cast<int>(blockIdx.x * blockDim.x + threadIdx.x);
  if (b >= B) return;
  const int n = __ldg(offsets + b + 1) - __ldg(offsets + b);
  int rank = 0;
  for (int o = 0; o < B; ++o) {
    const int m = __ldg(offsets + o + 1) - __ldg(offsets + o);
    rank += (m > n || (m == n && o < b)) ? 1 : 0;
  }
  order[rank] = b;
}

cudaError_t launch_cand_order(const CandArgs& a, cudaStream_t stream) {
  if (!a.order || a.B == 0) return cudaSuccess;
  cand_order<<<(a.B + 255) / 256, 256, 0, stream>>>(a.offsets, a.B, a.order);
  return cudaGetLastError();
}

cudaError_t launch_cand_sm100(const CandArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                              const CUtensorMap& tv, cudaStream_t stream) {
  if (a.B == 0 || a.C == 0) return cudaSuccess;
  const bool pos = a.rab_pos != nullptr, time = a.rab_time != nullptr;
  if (pos && time) return launch_t<true, true>(a, tq, tk, tv, stream);
  if (pos) return launch_t<true, false>(a, tq, tk, tv, stream);
  if (time) return launch_t<false, true>(a, tq, tk, tv, stream);
  return launch_t<false, false>(a, tq, tk, tv, stream);
}

}  // namespace hstu
