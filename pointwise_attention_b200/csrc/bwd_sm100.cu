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
// Two kernels, both deterministic (no floating-point atomics on dQ/dK/dV):
//  * hstu_bwd_dq_sm100   -- one CTA per (sequence, query tile, head); key
//    tiles 0..m: S = Q K^T and dA = dO V^T into TMEM, the epilogue turns them
//    into dS' (bf16, in TMEM), dQ += dS' K accumulates in TMEM.  It also sums
//    dS' along diagonals (position-bias gradient) and per time bucket.
//  * hstu_bwd_dkdv_sm100 -- one CTA per (sequence, key tile, head); query
//    tiles n..last: S^T = K Q^T and dA^T = V dO^T, the epilogue writes P'^T and
//    dS'^T over them in TMEM, dV += P'^T dO and dK += dS'^T Q accumulate.
// Roles: warp 0 TMA, warps 2..17 the epilogue (warp w: TMEM lane quarter w%4,
// 32-column quarter (w-2)/4), and the MMAs issued by two or three threads in
// warps 1, 18 and 19, one per independent accumulator chain: a tcgen05.mma
// costs its issuing thread about 110 cycles whatever its N up to 128, as long
// as the tensor core needs for the 128x128x16 step, so one thread issuing
// every GEMM of a tile would leave the tensor core idle most of the time.
#include <cuda_bf16.h>

#include <atomic>

#include "internal.h"
#include "ptx.cuh"
#include "tile_math.cuh"

namespace hstu {
namespace {

constexpr int kThreads = 640;
constexpr int kEpi = 512;
constexpr int kWarpB = 18;                   // second MMA issuer
constexpr int kWarpC = 19;                   // third MMA issuer (dQ kernel)
constexpr int kHalf = 16384;                 // 128 rows x 64 bf16
constexpr int kTile = 2 * kHalf;             // 128 x 128 bf16
constexpr int kTmemCols = 512;

constexpr uint32_t kIdescKK = idesc_bf16_f32(128, 128, false, false);  // A, B K-major
constexpr uint32_t kIdescTM = idesc_bf16_f32(128, 128, false, true);   // A TMEM, B MN-major

__device__ __forceinline__ void set_status(int* status, int bit) {
  if (status) atomicOr(status, bit);
}

// C[tmem] (+)= A (128 x 128, K-major tile in smem) * B (128 x 128, K-major tile)^T
__device__ __forceinline__ void mma_tile_kk(uint32_t d, uint32_t a_smem, uint32_t b_smem,
                                            bool accumulate) {
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const uint32_t off = (ks >> 2) * kHalf + (ks & 3) * 32;
    mma_ss(d, sw128_desc(a_smem + off, 16, 1024), sw128_desc(b_smem + off, 16, 1024), kIdescKK,
           (accumulate || ks > 0) ? 1u : 0u);
  }
}

// C[tmem] (+)= A (128 x 128 bf16 pairs in TMEM) * B, where B's 128 rows of
// 128 elements (row = reduction index) sit MN-major in a smem tile.
__device__ __forceinline__ void mma_tile_tm(uint32_t d, uint32_t a_tmem, uint32_t b_smem,
                                            bool accumulate) {
#pragma unroll
  for (int ks = 0; ks < 8; ++ks)
    mma_ts(d, a_tmem + 8u * ks, sw128_desc(b_smem + ks * 2048, kHalf, 1024), kIdescTM,
           (accumulate || ks > 0) ? 1u : 0u);
}

// From hx = (S + bias)/2 and t = tanh(hx):
//   sigma(x) = (1 + t)/2,  P' = SiLU(x) = hx (1 + t),
//   SiLU'(x) = sigma(x) (1 + x (1 - sigma(x))) = sigma(x) (1 + hx (1 - t)).
__device__ __forceinline__ float silu_grad_h(float hx, float t) {
  const float sg = fmaf(t, 0.5f, 0.5f);
  return sg * fmaf(hx, 1.0f - t, 1.0f);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Per-warp staging of one 32 x 32 block: 63 position-bias diagonals (fp32,
// halved) and the 32 column timestamps.
struct Stage {
  float w[64];
  long long ts[32];
};

// Time bias of one 32-column chunk for a row; `dir` = +1 when |dt| grows along
// the chunk (dK/dV kernel, columns are later queries), -1 when it shrinks (dQ
// kernel, columns are later keys).  With the chunk's timestamps sorted and
// dt of one sign over it, the bucket lies between the buckets of its two ends;
// when they differ by at most one, columns split at `split` (bisection).
struct ChunkT {
  int klo, khi;     // bucket before / from `split` on
  int split;
  bool simple;
};

template <int DIR>
__device__ __forceinline__ ChunkT chunk_time(long long my_ts, const long long* kts, bool sorted,
                                             const long long* thr, const signed char* first) {
  ChunkT c;
  c.split = 0;
  c.klo = c.khi = 0;
  // dt(c) = DIR > 0 ? kts[c] - my_ts : my_ts - kts[c], monotone in c
  const long long d0 = DIR > 0 ? kts[0] - my_ts : my_ts - kts[0];
  const long long d1 = DIR > 0 ? kts[31] - my_ts : my_ts - kts[31];
  c.simple = sorted && (DIR > 0 ? d0 >= 0 : d1 >= 0);
  if (c.simple) {
    const int k0 = time_bucket(d0, thr, first);
    const int k1 = time_bucket(d1, thr, first);
    c.simple = (k0 > k1 ? k0 - k1 : k1 - k0) <= 1;
    c.klo = k0;
    c.khi = k1;
    if (k0 != k1) {
      // first column whose bucket is k1: DIR>0 (increasing): dt >= thr[k1];
      // DIR<0 (decreasing): dt < thr[k0]
      int lo = 0, hi = 32;
#pragma unroll 1
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        const long long dm = DIR > 0 ? kts[mid] - my_ts : my_ts - kts[mid];
        const bool before = DIR > 0 ? dm < thr[k1] : dm >= thr[k0];
        if (before) lo = mid + 1; else hi = mid;
      }
      c.split = lo;
    } else {
      c.split = 32;
    }
  }
  return c;
}

// dS' of one 32-column chunk of the dQ kernel (rows = queries, columns =
// keys), its bf16 packing, and the bias-gradient accumulation.  MASK: the
// tile holds the diagonal or rows past the sequence end.
template <bool POS, bool TIME, bool MASK>
__device__ __forceinline__ void dq_chunk(const uint32_t (&sv)[32], const uint32_t (&dav)[32],
                                         const Stage* stg, int lane, int r, int c0, bool diag,
                                         bool row_ok, const ChunkT& ct, bool generic,
                                         long long my_ts, const long long* thr,
                                         const signed char* first, const float* rabt, float* win,
                                         float* s_dt, uint32_t (&packed)[16], float& t_lo,
                                         float& t_hi) {
  // Diagonal sums of the warp's 32 x 32 block without per-element atomics:
  // at column cl lane L reads column cl of lane (L + cl) mod 32, so every
  // element of diagonal L (row - column = L) or L - 32 passes through lane L.
  float dpos = 0.f, dneg = 0.f;
  // Per-element time buckets: the row's dS' is summed over runs of equal
  // bucket (with sorted timestamps the bucket only falls along the row) and a
  // run goes to the shared histogram when the bucket changes, instead of one
  // contended shared atomic per element.
  int run_k = -1;
  float run_s = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float ds2[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int cl = 2 * i + hh;
      const int c = c0 + cl;
      float hb = POS ? stg->w[lane - cl + 31] : 0.f;
      int kb = 0;
      if (TIME) {
        kb = generic ? time_bucket(my_ts - stg->ts[cl], thr, first)
                     : ((cl < ct.split) ? ct.klo : ct.khi);
        hb += rabt[kb];
      }
      const float hx = fmaf(__uint_as_float(sv[cl]), 0.5f, hb);
      const float t = tanh_approx(hx);
      float ds = __uint_as_float(dav[cl]) * silu_grad_h(hx, t);
      const bool masked = MASK && ((diag && c > r) || !row_ok);
      if (masked) ds = 0.f;
      ds2[hh] = ds;
      if (POS) {
        const float v = __shfl_sync(0xffffffffu, ds, (lane + cl) & 31);
        if (lane + cl < 32) dpos += v; else dneg += v;
      }
      if (TIME) {
        if (!generic) {
          if (cl < ct.split) t_lo += ds; else t_hi += ds;
        } else if (!masked) {
          if (kb != run_k) {
            if (run_k >= 0) atomicAdd(&s_dt[run_k], run_s);
            run_k = kb;
            run_s = 0.f;
          }
          run_s += ds;
        }
      }
    }
    packed[i] = pack_bf16(ds2[0], ds2[1]);
  }
  if (TIME && run_k >= 0) atomicAdd(&s_dt[run_k], run_s);
  if (POS) {
    // lane L holds diagonal L (window index r - c0 + 127 for this row's lane)
    // and diagonal L - 32 (index 32 lower); the latter is empty for lane 0.
    atomicAdd(&win[r - c0 + 127], dpos);
    if (lane > 0) atomicAdd(&win[r - c0 + 95], dneg);
  }
}

// P'^T and dS'^T of one 32-column chunk of the dK/dV kernel (rows = keys,
// columns = queries).  MASK: the diagonal tile or the sequence's last query tile.
template <bool POS, bool TIME, bool MASK>
__device__ __forceinline__ void dkv_chunk(const uint32_t (&sv)[32], const uint32_t (&dav)[32],
                                          const Stage* stg, int lane, int r, int c0, bool diag,
                                          int qlim, const ChunkT& ct, bool generic,
                                          long long my_ts, const long long* thr,
                                          const signed char* first, const float* rabt,
                                          uint32_t (&pk)[16], uint32_t (&dk)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float p2[2], d2[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int cl = 2 * i + hh;
      const int c = c0 + cl;
      float hb = POS ? stg->w[cl - lane + 31] : 0.f;
      if (TIME) {
        const int kb = generic ? time_bucket(stg->ts[cl] - my_ts, thr, first)
                               : ((cl < ct.split) ? ct.klo : ct.khi);
        hb += rabt[kb];
      }
      const float hx = fmaf(__uint_as_float(sv[cl]), 0.5f, hb);
      const float t = tanh_approx(hx);
      float p = fmaf(hx, t, hx);
      float ds = __uint_as_float(dav[cl]) * silu_grad_h(hx, t);
      if (MASK && ((diag && c < r) || c >= qlim)) {
        p = 0.f;
        ds = 0.f;
      }
      p2[hh] = p;
      d2[hh] = ds;
    }
    pk[i] = pack_bf16(p2[0], p2[1]);
    dk[i] = pack_bf16(d2[0], d2[1]);
  }
}

// ===================================================================== dQ
namespace dq {
constexpr int kOffQ = 0;
constexpr int kOffDO = kTile;
constexpr int kOffK = 2 * kTile;              // 2 stages
constexpr int kOffV = 4 * kTile;              // 2 stages
constexpr int kOffStage = 6 * kTile;          // 16 warps x Stage
constexpr int kOffWin = kOffStage + 16 * static_cast<int>(sizeof(Stage));   // 2 x 256 fp32
constexpr int kOffDT = kOffWin + 2 * 256 * 4;                                // 128 fp32
constexpr int kOffThr = kOffDT + 128 * 4;
constexpr int kOffFirst = kOffThr + kThrLen * 8;
constexpr int kOffRabT = kOffFirst + 64;
constexpr int kOffBar = kOffRabT + 128 * 4;
constexpr int kNumBars = 14;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmem = kOffMisc + 64 + 1024;

constexpr int B_QFULL = 0;     // Q and dO tiles
constexpr int B_KFULL = 1;     // +stage
constexpr int B_KEMPTY = 3;    // +stage (count 2: read by S and by dQ)
constexpr int B_VFULL = 5;     // +stage
constexpr int B_VEMPTY = 7;    // +stage
constexpr int B_SFULL = 9;     // S and dA of the current tile in TMEM (count 2)
constexpr int B_SFREE = 10;    // epilogue has read them (count kEpi)
constexpr int B_DSFULL = 11;   // +buffer, dS' written (count kEpi)
constexpr int B_DQFULL = 13;   // every MMA of the three issuers done (count 3)
constexpr uint32_t kColS = 0, kColDA = 128, kColDQ = 256, kColDS = 384;

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
  const int m = a.max_tiles - 1 - idx / a.B;
  const int b = idx % a.B;
  int s = __ldg(a.offsets + b);
  const int e_ = __ldg(a.offsets + b + 1);
  int n_b = e_ - s;
  if (s < 0 || n_b < 0 || e_ > a.T || n_b > a.max_seq_len || (POS && n_b > a.L)) {
    if (threadIdx.x == 0 && h == 0 && m == 0) set_status(a.status, kStatusBadOffsets);
    n_b = 0;
  }
  if (128 * m >= n_b) return;
  const int nt = m + 1;

  auto bar = [&](int i) { return sbase + kOffBar + 8u * i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  long long* s_thr = reinterpret_cast<long long*>(smem + kOffThr);
  signed char* s_first = reinterpret_cast<signed char*>(smem + kOffFirst);
  float* s_rabt = reinterpret_cast<float*>(smem + kOffRabT);
  float* s_win = reinterpret_cast<float*>(smem + kOffWin);
  float* s_dt = reinterpret_cast<float*>(smem + kOffDT);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      const bool epi = (i == B_SFREE || i == B_DSFULL || i == B_DSFULL + 1);
      uint32_t count = epi ? static_cast<uint32_t>(kEpi) : 1u;
      if (i == B_KEMPTY || i == B_KEMPTY + 1 || i == B_SFULL) count = 2;
      if (i == B_DQFULL) count = 3;
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
    if (POS && et < 512) s_win[et] = 0.f;
    if (TIME) {
      for (int i = et; i < kThrLen; i += kEpi) s_thr[i] = a.bt.thr[i];
      if (et < 64) s_first[et] = a.bt.first_k[et];
      if (et < a.nb) s_rabt[et] = 0.5f * __ldg(a.rab_time + static_cast<size_t>(h) * a.nb + et);
      if (et < 128) s_dt[et] = 0.f;
    }
  }
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
      const int row0 = s + 128 * m;
      mbar_arrive_expect_tx(bar(B_QFULL), 2 * kTile);
      tma_load_3d(sbase + kOffQ, &tm_q, bar(B_QFULL), 0, h, row0);
      tma_load_3d(sbase + kOffQ + kHalf, &tm_q, bar(B_QFULL), 64, h, row0);
      tma_load_3d(sbase + kOffDO, &tm_do, bar(B_QFULL), 0, h, row0);
      tma_load_3d(sbase + kOffDO + kHalf, &tm_do, bar(B_QFULL), 64, h, row0);
      int k_last[2] = {-1, -1}, v_last[2] = {-1, -1};
      bool ok = true;
      for (int n = 0; n < nt && ok; ++n) {
        const int st = n & 1, use = n >> 1;
        const int krow = s + 128 * n;
        if (use > 0) ok = mbar_wait(bar(B_KEMPTY + st), (use - 1) & 1, abort_flag);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(B_KFULL + st), kTile);
        tma_load_3d(sbase + kOffK + st * kTile, &tm_k, bar(B_KFULL + st), 0, h, krow);
        tma_load_3d(sbase + kOffK + st * kTile + kHalf, &tm_k, bar(B_KFULL + st), 64, h, krow);
        k_last[st] = use;
        if (use > 0) ok = mbar_wait(bar(B_VEMPTY + st), (use - 1) & 1, abort_flag);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(B_VFULL + st), kTile);
        tma_load_3d(sbase + kOffV + st * kTile, &tm_v, bar(B_VFULL + st), 0, h, krow);
        tma_load_3d(sbase + kOffV + st * kTile + kHalf, &tm_v, bar(B_VFULL + st), 64, h, krow);
        v_last[st] = use;
      }
      if (!ok) {
        set_status(a.status, kStatusTimeout);
        *abort_flag = 1;
        mbar_wait(bar(B_QFULL), 0, nullptr);
        for (int st = 0; st < 2; ++st) {
          if (k_last[st] >= 0) mbar_wait(bar(B_KFULL + st), k_last[st] & 1, nullptr);
          if (v_last[st] >= 0) mbar_wait(bar(B_VFULL + st), v_last[st] & 1, nullptr);
        }
      }
    }
  } else if (warp == 1 || warp == kWarpB || warp == kWarpC) {
    // ------------------------------------- MMA issuers: S (warp 1), dA, dQ
    if (lane == 0) {
      bool ok = true;
      if (warp == 1 || warp == kWarpB) {
        ok = mbar_wait(bar(B_QFULL), 0, abort_flag);
        for (int n = 0; n < nt && ok; ++n) {
          const int st = n & 1, use = n >> 1;
          ok = mbar_wait(bar((warp == 1 ? B_KFULL : B_VFULL) + st), use & 1, abort_flag);
          // S and dA of the previous tile have been read by the epilogue.
          if (ok && n > 0) ok = mbar_wait(bar(B_SFREE), (n - 1) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          if (warp == 1) {
            mma_tile_kk(tmem + kColS, sbase + kOffQ, sbase + kOffK + st * kTile, false);
            mma_commit(bar(B_KEMPTY + st));
          } else {
            mma_tile_kk(tmem + kColDA, sbase + kOffDO, sbase + kOffV + st * kTile, false);
            mma_commit(bar(B_VEMPTY + st));
          }
          mma_commit(bar(B_SFULL));
        }
      } else {
        for (int n = 0; n < nt && ok; ++n) {   // dQ += dS'(n) K_n
          ok = mbar_wait(bar(B_DSFULL + (n & 1)), (n >> 1) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          mma_tile_tm(tmem + kColDQ, tmem + kColDS + 64u * (n & 1),
                      sbase + kOffK + (n & 1) * kTile, n > 0);
          mma_commit(bar(B_KEMPTY + (n & 1)));
        }
      }
      if (!ok) {
        set_status(a.status, kStatusTimeout);
        *abort_flag = 1;
      }
      mma_commit(bar(B_DQFULL));
    }
  } else if (warp < kWarpB) {
    // ---------------------------------------------------------- epilogue
    const int q4 = warp & 3, cq = (warp - 2) >> 2;
    const int r = 32 * q4 + lane, et = threadIdx.x - 64;
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q4) << 16;
    const int i_loc = 128 * m + r;
    const bool row_ok = i_loc < n_b;
    const int t_row = s + (row_ok ? i_loc : 0);
    const float nrm = a.norm_len > 0 ? static_cast<float>(a.norm_len) : static_cast<float>(n_b);
    const float inv_n = 1.0f / nrm;
    const int Lw = 2 * a.L - 1;
    // Query rows past the sequence end (never stored) take the last token's
    // timestamp, which keeps their chunk plans on the cheap path.
    const long long my_ts = TIME ? a.timestamps[row_ok ? t_row : s + n_b - 1] : 0;
    Stage* stg = reinterpret_cast<Stage*>(smem + kOffStage) + (warp - 2);
    // This warp's block: rows 32 q4.., columns 32 cq..; diagonals
    // d = r - c in [32 q4 - 32 cq - 31, +31] (local index lane - cl + 31).
    const int dbase = 32 * q4 - 32 * cq - 31;
    float pw0 = 0.f, pw1 = 0.f;
    long long pt = 0;
    auto prefetch = [&](int n) {
      if (POS) {
        const int t0 = 128 * (m - n) + dbase + lane + a.L - 1;
        const float* tab = a.rab_pos + static_cast<size_t>(h) * Lw;
        pw0 = (t0 >= 0 && t0 < Lw) ? __ldg(tab + t0) : 0.f;
        pw1 = (lane < 31 && t0 + 32 >= 0 && t0 + 32 < Lw) ? __ldg(tab + t0 + 32) : 0.f;
      }
      if (TIME) {
        const int j = 128 * n + 32 * cq + lane;
        pt = a.timestamps[s + (j < n_b ? j : n_b - 1)];
      }
    };
    bool sorted = true;
    auto stage = [&]() {
      if (POS) {
        stg->w[lane] = 0.5f * pw0;
        stg->w[32 + lane] = 0.5f * pw1;
      }
      if (TIME) {
        stg->ts[lane] = pt;
        const long long nx = __shfl_down_sync(0xffffffffu, pt, 1);
        sorted = !__any_sync(0xffffffffu, lane < 31 && nx < pt);
      }
      __syncwarp();
    };
    prefetch(0);
    stage();
    bool ok = true;
    for (int n = 0; n < nt; ++n) {
      if (n + 1 < nt) prefetch(n + 1);
      if (ok) ok = mbar_wait(bar(B_SFULL), n & 1, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      float* win = s_win + 256 * (n & 1);
      if (ok) {
        tc_fence_after();
        uint32_t sv[32], dav[32];
        tmem_ld32_nowait(tmem + lane_addr + kColS + 32u * cq, sv);
        tmem_ld32_nowait(tmem + lane_addr + kColDA + 32u * cq, dav);
        tmem_wait_ld_dep(sv);
        tmem_wait_ld_dep(dav);
        tc_fence_before();
        mbar_arrive(bar(B_SFREE));
        const bool diag = (n == m);
        ChunkT ct{};
        bool generic = false;
        if (TIME) {
          ct = chunk_time<-1>(my_ts, stg->ts, sorted, s_thr, s_first);
          generic = !__all_sync(0xffffffffu, ct.simple);
        }
        float t_lo = 0.f, t_hi = 0.f;      // d_rab_time partial sums (simple path)
        uint32_t packed[16];
        if (diag || !__all_sync(0xffffffffu, row_ok))
          dq_chunk<POS, TIME, true>(sv, dav, stg, lane, r, 32 * cq, diag, row_ok, ct, generic,
                                    my_ts, s_thr, s_first, s_rabt, win, s_dt, packed, t_lo, t_hi);
        else
          dq_chunk<POS, TIME, false>(sv, dav, stg, lane, r, 32 * cq, diag, row_ok, ct, generic,
                                     my_ts, s_thr, s_first, s_rabt, win, s_dt, packed, t_lo,
                                     t_hi);
        if (TIME && !generic) {
          if (t_lo != 0.f) atomicAdd(&s_dt[ct.klo], t_lo);
          if (t_hi != 0.f) atomicAdd(&s_dt[ct.khi], t_hi);
        }
        tmem_st16(tmem + lane_addr + kColDS + 64u * (n & 1) + 16u * cq, packed);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(B_DSFULL + (n & 1)));
      }
      if (n + 1 < nt) stage();
      // Every epilogue warp has added its dS' of tile n to the diagonal sums.
      named_bar_sync(1, kEpi);
      if (POS && et < 255) {
        const float v = win[et];
        const int tbl = 128 * (m - n) + et - 127 + a.L - 1;
        if (v != 0.f && tbl >= 0 && tbl < Lw)
          atomicAdd(a.d_rab_pos + static_cast<size_t>(h) * Lw + tbl, v * inv_n);
        win[et] = 0.f;
      }
    }
    // dQ = (1/N) sum dS' K
    if (ok) ok = mbar_wait(bar(B_DQFULL), 0, abort_flag);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) {
      set_status(a.status, kStatusTimeout);
      *abort_flag = 1;
    }
    tc_fence_after();
    {
      uint32_t qv[32];
      tmem_ld32_nowait(tmem + lane_addr + kColDQ + 32u * cq, qv);
      tmem_wait_ld_dep(qv);
      if (ok && row_ok) {
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.dq) +
                                              (static_cast<size_t>(t_row) * a.H + h) * 128 +
                                              32 * cq);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint4 o;
          o.x = pack_bf16(__uint_as_float(qv[8 * i + 0]) * inv_n, __uint_as_float(qv[8 * i + 1]) * inv_n);
          o.y = pack_bf16(__uint_as_float(qv[8 * i + 2]) * inv_n, __uint_as_float(qv[8 * i + 3]) * inv_n);
          o.z = pack_bf16(__uint_as_float(qv[8 * i + 4]) * inv_n, __uint_as_float(qv[8 * i + 5]) * inv_n);
          o.w = pack_bf16(__uint_as_float(qv[8 * i + 6]) * inv_n, __uint_as_float(qv[8 * i + 7]) * inv_n);
          dst[i] = o;
        }
      }
    }
    if (TIME) {
      named_bar_sync(1, kEpi);
      if (et < a.nb && s_dt[et] != 0.f)
        atomicAdd(a.d_rab_time + static_cast<size_t>(h) * a.nb + et, s_dt[et] * inv_n);
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if (lane == 0) mbar_wait(bar(B_DQFULL), 0, nullptr);
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}
}  // namespace dq

// =================================================================== dK, dV
namespace dkv {
constexpr int kOffK = 0;
constexpr int kOffV = kTile;
constexpr int kOffQ = 2 * kTile;              // 2 stages
constexpr int kOffDO = 4 * kTile;             // 2 stages
constexpr int kOffStage = 6 * kTile;
constexpr int kOffThr = kOffStage + 16 * static_cast<int>(sizeof(Stage));
constexpr int kOffFirst = kOffThr + kThrLen * 8;
constexpr int kOffRabT = kOffFirst + 64;
constexpr int kOffBar = kOffRabT + 128 * 4;
constexpr int kNumBars = 10;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmem = kOffMisc + 64 + 1024;

constexpr int B_KVFULL = 0;
constexpr int B_QFULL = 1;     // +stage: Q and dO tiles
constexpr int B_QEMPTY = 3;    // +stage (count 2: one per issuer)
constexpr int B_SFULL = 5;     // S^T and dA^T in TMEM (count 2)
constexpr int B_PFULL = 6;     // P'^T and dS'^T written over them (count kEpi)
constexpr int B_PDDONE = 7;    // dV/dK MMAs of the tile done (count 2)
constexpr int B_OUT = 8;       // every MMA of both issuers done (count 2)
// S^T at [0,128) with P'^T over [0,64); dA^T at [128,256) with dS'^T over [128,192)
constexpr uint32_t kColS = 0, kColDA = 128, kColDV = 256, kColDK = 384;

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
  int s = __ldg(a.offsets + b);
  const int e_ = __ldg(a.offsets + b + 1);
  int n_b = e_ - s;
  if (s < 0 || n_b < 0 || e_ > a.T || n_b > a.max_seq_len || (POS && n_b > a.L)) n_b = 0;
  if (128 * n >= n_b) return;
  const int mt_b = (n_b + 127) / 128;         // query tiles of this sequence
  const int nq = mt_b - n;                    // query tiles n .. mt_b-1

  auto bar = [&](int i) { return sbase + kOffBar + 8u * i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  long long* s_thr = reinterpret_cast<long long*>(smem + kOffThr);
  signed char* s_first = reinterpret_cast<signed char*>(smem + kOffFirst);
  float* s_rabt = reinterpret_cast<float*>(smem + kOffRabT);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      uint32_t count = i == B_PFULL ? static_cast<uint32_t>(kEpi) : 1u;
      if (i == B_QEMPTY || i == B_QEMPTY + 1 || i == B_SFULL || i == B_PDDONE || i == B_OUT)
        count = 2;
      mbar_init(bar(i), count);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sbase + kOffMisc, kTmemCols);
    tmem_relinquish();
  }
  if (TIME && warp >= 2 && warp < kWarpB) {
    const int et = threadIdx.x - 64;
    for (int i = et; i < kThrLen; i += kEpi) s_thr[i] = a.bt.thr[i];
    if (et < 64) s_first[et] = a.bt.first_k[et];
    if (et < a.nb) s_rabt[et] = 0.5f * __ldg(a.rab_time + static_cast<size_t>(h) * a.nb + et);
  }
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
      const int krow = s + 128 * n;
      mbar_arrive_expect_tx(bar(B_KVFULL), 2 * kTile);
      tma_load_3d(sbase + kOffK, &tm_k, bar(B_KVFULL), 0, h, krow);
      tma_load_3d(sbase + kOffK + kHalf, &tm_k, bar(B_KVFULL), 64, h, krow);
      tma_load_3d(sbase + kOffV, &tm_v, bar(B_KVFULL), 0, h, krow);
      tma_load_3d(sbase + kOffV + kHalf, &tm_v, bar(B_KVFULL), 64, h, krow);
      int q_last[2] = {-1, -1};
      bool ok = true;
      for (int it = 0; it < nq && ok; ++it) {
        const int st = it & 1, use = it >> 1;
        const int qrow = s + 128 * (n + it);
        if (use > 0) ok = mbar_wait(bar(B_QEMPTY + st), (use - 1) & 1, abort_flag);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(B_QFULL + st), 2 * kTile);
        tma_load_3d(sbase + kOffQ + st * kTile, &tm_q, bar(B_QFULL + st), 0, h, qrow);
        tma_load_3d(sbase + kOffQ + st * kTile + kHalf, &tm_q, bar(B_QFULL + st), 64, h, qrow);
        tma_load_3d(sbase + kOffDO + st * kTile, &tm_do, bar(B_QFULL + st), 0, h, qrow);
        tma_load_3d(sbase + kOffDO + st * kTile + kHalf, &tm_do, bar(B_QFULL + st), 64, h, qrow);
        q_last[st] = use;
      }
      if (!ok) {
        set_status(a.status, kStatusTimeout);
        *abort_flag = 1;
        mbar_wait(bar(B_KVFULL), 0, nullptr);
        for (int st = 0; st < 2; ++st)
          if (q_last[st] >= 0) mbar_wait(bar(B_QFULL + st), q_last[st] & 1, nullptr);
      }
    }
  } else if (warp == 1 || warp == kWarpB) {
    // ------------------- MMA issuers: S^T then dV (warp 1), dA^T then dK
    if (lane == 0) {
      const bool first = (warp == 1);
      bool ok = mbar_wait(bar(B_KVFULL), 0, abort_flag);
      for (int it = 0; it < nq && ok; ++it) {
        const int st = it & 1;
        ok = mbar_wait(bar(B_QFULL + st), (it >> 1) & 1, abort_flag);
        // P'^T / dS'^T of the previous tile live in the S / dA columns: their
        // dV / dK products (both issuers') must be finished before S^T / dA^T
        // are rewritten.
        if (ok && it > 0) ok = mbar_wait(bar(B_PDDONE), (it - 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t qa = sbase + kOffQ + st * kTile, da = sbase + kOffDO + st * kTile;
        if (first)
          mma_tile_kk(tmem + kColS, sbase + kOffK, qa, false);   // S^T = K Q^T
        else
          mma_tile_kk(tmem + kColDA, sbase + kOffV, da, false);  // dA^T = V dO^T
        mma_commit(bar(B_SFULL));
        ok = mbar_wait(bar(B_PFULL), it & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        if (first)
          mma_tile_tm(tmem + kColDV, tmem + kColS, da, it > 0);  // dV += P'^T dO
        else
          mma_tile_tm(tmem + kColDK, tmem + kColDA, qa, it > 0); // dK += dS'^T Q
        mma_commit(bar(B_QEMPTY + st));
        mma_commit(bar(B_PDDONE));
      }
      if (!ok) {
        set_status(a.status, kStatusTimeout);
        *abort_flag = 1;
      }
      mma_commit(bar(B_OUT));
    }
  } else if (warp < kWarpB) {
    // ---------------------------------------------------------- epilogue
    const int q4 = warp & 3, cq = (warp - 2) >> 2;
    const int r = 32 * q4 + lane, et = threadIdx.x - 64;
    (void)et;
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q4) << 16;
    const int j_loc = 128 * n + r;                  // this thread's key
    const bool row_ok = j_loc < n_b;
    const int t_row = s + (row_ok ? j_loc : 0);
    const float nrm = a.norm_len > 0 ? static_cast<float>(a.norm_len) : static_cast<float>(n_b);
    const float inv_n = 1.0f / nrm;
    const int Lw = 2 * a.L - 1;
    const long long my_ts = TIME ? a.timestamps[t_row] : 0;
    Stage* stg = reinterpret_cast<Stage*>(smem + kOffStage) + (warp - 2);
    // This warp's block: key rows 32 q4.., query columns 32 cq..; index
    // i - j = 128 (m - n) + c - r, c - r in [32 cq - 32 q4 - 31, +31]
    // (local index cl - lane + 31).
    const int dbase = 32 * cq - 32 * q4 - 31;
    float pw0 = 0.f, pw1 = 0.f;
    long long pt = 0;
    auto prefetch = [&](int it) {
      const int mq = n + it;
      if (POS) {
        const int t0 = 128 * (mq - n) + dbase + lane + a.L - 1;
        const float* tab = a.rab_pos + static_cast<size_t>(h) * Lw;
        pw0 = (t0 >= 0 && t0 < Lw) ? __ldg(tab + t0) : 0.f;
        pw1 = (lane < 31 && t0 + 32 >= 0 && t0 + 32 < Lw) ? __ldg(tab + t0 + 32) : 0.f;
      }
      if (TIME) {
        const int i = 128 * mq + 32 * cq + lane;
        pt = a.timestamps[s + (i < n_b ? i : n_b - 1)];
      }
    };
    bool sorted = true;
    auto stage = [&]() {
      if (POS) {
        stg->w[lane] = 0.5f * pw0;
        stg->w[32 + lane] = 0.5f * pw1;
      }
      if (TIME) {
        stg->ts[lane] = pt;
        const long long nx = __shfl_down_sync(0xffffffffu, pt, 1);
        sorted = !__any_sync(0xffffffffu, lane < 31 && nx < pt);
      }
      __syncwarp();
    };
    prefetch(0);
    stage();
    bool ok = true;
    for (int it = 0; it < nq; ++it) {
      const int mq = n + it;
      if (it + 1 < nq) prefetch(it + 1);
      if (ok) ok = mbar_wait(bar(B_SFULL), it & 1, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      uint32_t pk[16], dk[16];
      if (ok) {
        tc_fence_after();
        uint32_t sv[32], dav[32];
        tmem_ld32_nowait(tmem + lane_addr + kColS + 32u * cq, sv);
        tmem_ld32_nowait(tmem + lane_addr + kColDA + 32u * cq, dav);
        tmem_wait_ld_dep(sv);
        tmem_wait_ld_dep(dav);
        const bool diag = (mq == n);
        const int qlim = n_b - 128 * mq;          // valid query columns c < qlim
        ChunkT ct{};
        bool generic = false;
        if (TIME) {
          ct = chunk_time<+1>(my_ts, stg->ts, sorted, s_thr, s_first);
          generic = !__all_sync(0xffffffffu, ct.simple);
        }
        if (diag || qlim < 128)
          dkv_chunk<POS, TIME, true>(sv, dav, stg, lane, r, 32 * cq, diag, qlim, ct, generic,
                                     my_ts, s_thr, s_first, s_rabt, pk, dk);
        else
          dkv_chunk<POS, TIME, false>(sv, dav, stg, lane, r, 32 * cq, diag, qlim, ct, generic,
                                      my_ts, s_thr, s_first, s_rabt, pk, dk);
      }
      // Every warp has read its S^T / dA^T columns before any is overwritten.
      named_bar_sync(1, kEpi);
      if (ok) {
        tmem_st16(tmem + lane_addr + kColS + 16u * cq, pk);
        tmem_st16(tmem + lane_addr + kColDA + 16u * cq, dk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(B_PFULL));
      }
      if (it + 1 < nq) stage();
    }
    if (ok) ok = mbar_wait(bar(B_OUT), 0, abort_flag);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) {
      set_status(a.status, kStatusTimeout);
      *abort_flag = 1;
    }
    tc_fence_after();
    uint32_t vv[32], kv[32];
    tmem_ld32_nowait(tmem + lane_addr + kColDV + 32u * cq, vv);
    tmem_ld32_nowait(tmem + lane_addr + kColDK + 32u * cq, kv);
    tmem_wait_ld_dep(vv);
    tmem_wait_ld_dep(kv);
    if (ok && row_ok) {
      const size_t off = (static_cast<size_t>(t_row) * a.H + h) * 128 + 32 * cq;
      uint4* dvp = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.dv) + off);
      uint4* dkp = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.dk) + off);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint4 o;
        o.x = pack_bf16(__uint_as_float(vv[8 * i + 0]) * inv_n, __uint_as_float(vv[8 * i + 1]) * inv_n);
        o.y = pack_bf16(__uint_as_float(vv[8 * i + 2]) * inv_n, __uint_as_float(vv[8 * i + 3]) * inv_n);
        o.z = pack_bf16(__uint_as_float(vv[8 * i + 4]) * inv_n, __uint_as_float(vv[8 * i + 5]) * inv_n);
        o.w = pack_bf16(__uint_as_float(vv[8 * i + 6]) * inv_n, __uint_as_float(vv[8 * i + 7]) * inv_n);
        dvp[i] = o;
        o.x = pack_bf16(__uint_as_float(kv[8 * i + 0]) * inv_n, __uint_as_float(kv[8 * i + 1]) * inv_n);
        o.y = pack_bf16(__uint_as_float(kv[8 * i + 2]) * inv_n, __uint_as_float(kv[8 * i + 3]) * inv_n);
        o.z = pack_bf16(__uint_as_float(kv[8 * i + 4]) * inv_n, __uint_as_float(kv[8 * i + 5]) * inv_n);
        o.w = pack_bf16(__uint_as_float(kv[8 * i + 6]) * inv_n, __uint_as_float(kv[8 * i + 7]) * inv_n);
        dkp[i] = o;
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

// `configured` caches, per device, that the kernel's shared-memory opt-in has
// been set.  Host threads may launch concurrently: the flag is atomic, and two
// threads that both see it clear just set the same attribute twice.
template <typename K>
cudaError_t launch_plain(K kernel, int smem, unsigned grid, const CUtensorMap* maps,
                         const BwdArgs& a, cudaStream_t stream, std::atomic<bool>* configured) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  const bool cached = dev >= 0 && dev < 64;
  if (!cached || !configured[dev].load(std::memory_order_acquire)) {
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    if (cached) configured[dev].store(true, std::memory_order_release);
  }
  kernel<<<grid, kThreads, smem, stream>>>(maps[0], maps[1], maps[2], maps[3], a);
  return cudaGetLastError();
}

template <bool POS, bool TIME>
cudaError_t launch_variant(const BwdArgs& a, const CUtensorMap* maps, cudaStream_t stream) {
  static std::atomic<bool> conf_dq[64], conf_dkv[64];   // zero-initialised: false
  const unsigned grid = static_cast<unsigned>(a.H) * static_cast<unsigned>(a.B) *
                        static_cast<unsigned>(a.max_tiles);
  cudaError_t err = launch_plain(dq::hstu_bwd_dq_sm100<POS, TIME>, dq::kSmem, grid, maps, a,
                                 stream, conf_dq);
  if (err != cudaSuccess) return err;
  return launch_plain(dkv::hstu_bwd_dkdv_sm100<POS, TIME>, dkv::kSmem, grid, maps, a, stream,
                      conf_dkv);
}

}  // namespace

// maps: q, k, v, dO ([T, H, 128] bf16, 128-row boxes).  The LN/gate part (dO,
// dU) must already be in a.dO / a.du.
cudaError_t launch_bwd_attn_bf16_sm100(const BwdArgs& a, const CUtensorMap* maps,
                                       cudaStream_t stream) {
  if (a.B == 0 || a.max_tiles == 0) return cudaSuccess;
  const bool pos = a.rab_pos != nullptr, tim = a.rab_time != nullptr;
  if (pos && tim) return launch_variant<true, true>(a, maps, stream);
  if (pos) return launch_variant<true, false>(a, maps, stream);
  if (tim) return launch_variant<false, true>(a, maps, stream);
  return launch_variant<false, false>(a, maps, stream);
}

}  // namespace hstu
