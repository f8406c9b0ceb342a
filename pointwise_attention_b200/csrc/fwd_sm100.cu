// fwd_sm100.cu -- bf16 forward of HSTU causal pointwise aggregated attention
// on sm_100a: TMA-staged Q/K/V tiles, tcgen05 MMAs with TMEM accumulators,
// a register epilogue for bias + SiLU + 1/N + causal mask between the two
// MMAs, and the LayerNorm-over-heads + SiLU(U) gate fused into the store.
//
// Operation: "HSTU (Generative Recommender)" model card, Exported PyTorch,
// HSTUBlock.forward (silu(q k^T)/t, tril, attn @ v, gate by silu(u));
// relative position / time bias: "HSTU Hierarchical Sequential Transduction
// Units", §1 and §3; post-pooling normalisation then U gate: the HSTU
// reproduction note's flowchart.
//
// Work decomposition.  One CTA computes one (sequence b, query tile m, head h):
// 128 query rows against key tiles n = 0..m (tiles above the diagonal are
// skipped; only the diagonal tile is masked).  The H CTAs of one (b, m) form a
// thread-block cluster so the LayerNorm over the concatenated heads can
// exchange per-row partial sums through distributed shared memory (st.async).
// Clusters enumerate (m descending, b), so the CTAs with the most key tiles are
// dispatched first (the cost of a tile depends on m only).
//
// Roles (576 threads): warp 0 issues TMA, warp 1 allocates TMEM and issues the
// MMAs (one thread), warps 2..17 form the epilogue in two teams of 8 warps:
// team t = (w-2)/8 turns the S tiles n = t, t+2, t+4, ... (S buffer t) into P,
// so the two teams overlap each other's waits; warp w owns TMEM lane quarter
// w%4 (rows 32*(w%4) ..) and column half ((w-2)/4)%2 (64 columns) of its team's
// tiles.  Each warp stages the position-bias diagonals and key timestamps of
// its own 32x64 block in a private buffer, fetched from global memory one tile
// ahead.  Waiting on S(n) also covers P buffer reuse: the MMA thread commits
// S(n) after issuing P(n-2).V, and a commit tracks every earlier MMA.
//
// TMEM (512 columns): S0 [0,128) S1 [128,256) O [256,384) P0 [384,448)
// P1 [448,512).  S = Q K^T is fp32; P' = SiLU(S+bias) is packed bf16 pairs and
// is the A operand (from TMEM) of O' += P' V; O = O' / N in the epilogue.
//
// Every tcgen05.ld/st is warp-collective (.sync.aligned): they are issued by
// all 32 lanes with warp-uniform control flow; only global accesses are
// predicated per row.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"
#include "tile_math.cuh"

namespace hstu {
namespace {

constexpr int kThreads = 576;
constexpr int kEpiThreads = 512;
constexpr int kColGroups = 4;               // epilogue warpgroups, 32 columns each
constexpr int kRows = 128;                  // query rows per tile
constexpr int kCols = 128;                  // keys per tile
constexpr int kHalf = 16384;                // 128 rows x 64 bf16 (one 128B-swizzle slab)
constexpr int kTile = 2 * kHalf;            // 128 x 128 bf16
constexpr int kKStages = 3;                 // K tiles in flight (S = Q K^T needs them first)
constexpr int kVStages = 2;                 // V tiles in flight (P.V comes a tile later)

// shared-memory map (byte offsets from a 1024-aligned base)
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kTile;                    // kKStages tiles
constexpr int kOffV = kOffK + kKStages * kTile;         // kVStages tiles
// Per epilogue warp: 96 fp32 half position-bias values (the 95 diagonals its
// 32x64 block touches) and 64 int64 key timestamps.
constexpr int kWarpStage = 96 * 4 + 64 * 8;             // bytes per warp
constexpr int kOffWarp = kOffV + kVStages * kTile;
constexpr int kOffThr = kOffWarp + 16 * kWarpStage;     // kThrLen int64 thresholds
constexpr int kOffFirst = kOffThr + kThrLen * 8;        // 64 int8 first bucket per octave
constexpr int kOffRabT = kOffFirst + 64;                // 128 fp32 half time-bias row
// LayerNorm reduction: per round, [4 column groups][128 rows] local partials
// and [8 heads][128 rows] cluster exchange slots.
constexpr int kOffRed = kOffRabT + 128 * 4;
constexpr int kRedBytes = 2 * (kColGroups * 128 + 8 * 128) * 4;
constexpr int kOffBar = kOffRed + kRedBytes;            // mbarriers (8 B each)
constexpr int kNumBars = 16;
constexpr int kOffMisc = kOffBar + kNumBars * 8;        // tmem base, abort flag, 2 LN barriers
constexpr int kSmemBytes = kOffMisc + 64 + 1024;        // + alignment slack

// barrier indices
constexpr int B_QFULL = 0;
constexpr int B_KFULL = 1;    // +K stage
constexpr int B_KEMPTY = 4;   // +K stage
constexpr int B_VFULL = 7;    // +V stage
constexpr int B_VEMPTY = 9;   // +V stage
constexpr int B_SFULL = 11;   // +buffer
constexpr int B_PFULL = 13;   // +buffer
constexpr int B_OFULL = 15;
constexpr int kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColO = 256, kColP0 = 384;

constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false, false);   // Q (K-major) x K (K-major)
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, false, true);   // P (TMEM) x V (MN-major)

__device__ __forceinline__ void set_status(int* status, int bit) {
  if (status) atomicOr(status, bit);
}

struct EpiCtx {
  const float* win;           // warp's half position bias: element (lane, cl) -> win[lane - cl + 31]
  const long long* kts;       // warp's 32 key timestamps
  const long long* thr;       // bucket thresholds
  const signed char* first;   // first bucket per octave
  const float* rabt;          // half time bias per bucket
  long long my_ts;            // this row's timestamp
  bool chunk_sorted;          // the warp's key timestamps are non-decreasing
  float inv_n;                // 1 / N_b
  int r;                      // row in the tile
  int lane;
};

// Time bias of a 32-column chunk for this row.  With the tile's key timestamps
// sorted and the row not before the chunk's last key, |t_i - t_j| falls along
// the chunk, so the bucket lies between the buckets k0 >= k1 of its two ends;
// when they differ by at most one, the columns before `split` (bisection) take
// k0 and the rest k1 ("simple").  Otherwise every element takes the full search.
struct ChunkTime {
  float hi, lo;     // half time bias of buckets k0 and k1
  int split;        // columns [0, split) take `hi`
  bool simple;
};

__device__ __forceinline__ ChunkTime chunk_time(const EpiCtx& e) {
  ChunkTime ct;
  ct.hi = ct.lo = 0.f;
  ct.split = 0;
  const long long d0 = e.my_ts - e.kts[0];
  const long long d1 = e.my_ts - e.kts[31];
  ct.simple = e.chunk_sorted && d1 >= 0;
  if (ct.simple) {
    const int k0 = time_bucket(d0, e.thr, e.first);
    const int k1 = time_bucket(d1, e.thr, e.first);
    ct.simple = (k0 - k1) <= 1;
    ct.hi = e.rabt[k0];
    ct.lo = e.rabt[k1];
    if (k0 != k1) {
      // columns c with t_i - t_c >= thr[k0]  <=>  t_c <= t_i - thr[k0]
      const long long lim = e.my_ts - e.thr[k0];
      int lo = 0, hi = 32;   // first column with kts > lim
#pragma unroll 1
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (e.kts[mid] <= lim) lo = mid + 1; else hi = mid;
      }
      ct.split = lo;
    }
  }
  return ct;
}

// P' = N * SiLU(S + bias) / N for two adjacent columns, packed as bf16x2:
//   hx = (S + bias)/2,  P' = hx (1 + tanh(hx)) = SiLU(S + bias).
// hx is rounded to bf16, tanh and the fused multiply-add run on bf16 pairs
// (one MUFU operation per two elements); the 1/N factor is applied to O in
// fp32 after the A.V accumulation instead of to every element of P.
__device__ __forceinline__ uint32_t p_pair(float hx0, float hx1) {
  __nv_bfloat162 h2 = __floats2bfloat162_rn(hx0, hx1);   // .x (low half) = hx0
  const uint32_t hv = *reinterpret_cast<uint32_t*>(&h2);
  uint32_t tv, pv;
  asm("tanh.approx.bf16x2 %0, %1;" : "=r"(tv) : "r"(hv));
  asm("fma.rn.bf16x2 %0, %1, %2, %1;" : "=r"(pv) : "r"(hv), "r"(tv));
  return pv;
}

// MODE 0: position bias only (or none); 1: plus a per-row time bias constant
// (`lo`); 2: plus the per-row two-value split; 3: per-element bucket search.
template <bool POS, int MODE, bool DIAG>
__device__ __forceinline__ void chunk_to_p(const uint32_t (&sraw)[32], int c0, const EpiCtx& e,
                                           const ChunkTime& ct, uint32_t (&packed)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float hx[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int cl = 2 * i + hh;
      float hb = POS ? e.win[e.lane - cl + 31] : 0.f;
      if (MODE == 1) hb += ct.lo;
      if (MODE == 2) hb += (cl < ct.split) ? ct.hi : ct.lo;
      if (MODE == 3) hb += e.rabt[time_bucket(e.my_ts - e.kts[cl], e.thr, e.first)];
      hx[hh] = fmaf(__uint_as_float(sraw[cl]), 0.5f, hb);
    }
    uint32_t pv = p_pair(hx[0], hx[1]);
    if (DIAG) {   // causal mask: column c > row r is exactly zero
      const int c = c0 + 2 * i;
      const uint32_t keep = (c > e.r ? 0u : 0x0000FFFFu) | (c + 1 > e.r ? 0u : 0xFFFF0000u);
      pv &= keep;
    }
    packed[i] = pv;
  }
}

// Chunk k (32 columns) of this thread's 64 columns -> 16 packed P words.
template <bool POS, bool TIME, bool DIAG>
__device__ __forceinline__ void chunk_p(const uint32_t (&sv)[32], int c0, const EpiCtx& e,
                                        uint32_t (&packed)[16]) {
  if (!TIME) {
    chunk_to_p<POS, 0, DIAG>(sv, c0, e, ChunkTime{}, packed);
  } else {
    const ChunkTime ct = chunk_time(e);
    // Warp-uniform choice of the element loop.
    if (!__all_sync(0xffffffffu, ct.simple)) {
      chunk_to_p<POS, 3, DIAG>(sv, c0, e, ct, packed);
    } else if (__any_sync(0xffffffffu, ct.split != 0)) {
      chunk_to_p<POS, 2, DIAG>(sv, c0, e, ct, packed);
    } else {
      chunk_to_p<POS, 1, DIAG>(sv, c0, e, ct, packed);
    }
  }
}

// This thread's 64 columns (col0 .. col0+63) of the S tile -> P in TMEM.
// `wv` holds the warp's 96 staged diagonals, `kts` its 64 key timestamps.
template <bool POS, bool TIME, bool DIAG>
__device__ __forceinline__ void tile_to_p(uint32_t s_addr, uint32_t p_addr, int col0,
                                          EpiCtx& e, const float* wv, const long long* kts,
                                          bool sorted0, bool sorted1) {
  uint32_t sv[32];
  uint32_t packed[16];
  // chunk 0: element (lane, cl) uses diagonal index lane - cl + 63
  tmem_ld32_nowait(s_addr + col0, sv);
  tmem_wait_ld_dep(sv);
  e.win = wv + 32;
  e.kts = kts;
  e.chunk_sorted = sorted0;
  chunk_p<POS, TIME, DIAG>(sv, col0, e, packed);
  tmem_st16(p_addr + col0 / 2, packed);
  // chunk 1: index lane - cl + 31
  tmem_ld32_nowait(s_addr + col0 + 32, sv);
  tmem_wait_ld_dep(sv);
  e.win = wv;
  e.kts = kts + 32;
  e.chunk_sorted = sorted1;
  chunk_p<POS, TIME, DIAG>(sv, col0 + 32, e, packed);
  tmem_st16(p_addr + col0 / 2 + 16, packed);
}

template <bool POS, bool TIME>
__global__ void __launch_bounds__(kThreads, 1)
    hstu_fwd_bf16_sm100(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ FwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // blockIdx.x = (cluster index) * H + head; the head is the rank in the cluster.
  const int h = static_cast<int>(blockIdx.x % static_cast<unsigned>(a.H));
  const int idx = static_cast<int>(blockIdx.x / static_cast<unsigned>(a.H));
  const int m = a.max_tiles - 1 - idx / a.B;
  const int b = idx % a.B;

  // Sequence bounds; inconsistent offsets make the sequence empty and are reported.
  int s = __ldg(a.offsets + b);
  int e = __ldg(a.offsets + b + 1);
  int n_b = e - s;
  if (s < 0 || n_b < 0 || e > a.T || n_b > a.max_seq_len || (POS && n_b > a.L)) {
    if (threadIdx.x == 0 && h == 0 && m == 0) set_status(a.status, kStatusBadOffsets);
    n_b = 0;
  }
  if (kRows * m >= n_b) return;               // whole cluster leaves together
  const int nt = m + 1;                       // key tiles 0..m

  auto bar = [&](int i) { return sbase + kOffBar + 8u * i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  const uint32_t bar_red0 = sbase + kOffMisc + 16;   // 8-byte aligned slots in misc
  const uint32_t bar_red1 = sbase + kOffMisc + 24;

  long long* s_thr = reinterpret_cast<long long*>(smem + kOffThr);
  signed char* s_first = reinterpret_cast<signed char*>(smem + kOffFirst);
  float* s_rabt = reinterpret_cast<float*>(smem + kOffRabT);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i)
      mbar_init(bar(i), (i == B_PFULL || i == B_PFULL + 1)
                            ? static_cast<uint32_t>(kEpiThreads / 2)   // one team
                            : 1u);
    mbar_init(bar_red0, 1);
    mbar_init(bar_red1, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sbase + kOffMisc, kTmemCols);
    tmem_relinquish();
  }
  if (TIME && warp >= 2) {
    const int et = threadIdx.x - 64;
    for (int i = et; i < kThrLen; i += kEpiThreads) s_thr[i] = a.bt.thr[i];
    if (et < 64) s_first[et] = a.bt.first_k[et];
    if (et < a.nb) s_rabt[et] = 0.5f * __ldg(a.rab_time + static_cast<size_t>(h) * a.nb + et);
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Every CTA of the cluster has initialised its barriers before any remote access.
  cluster_arrive();
  cluster_wait();
  const uint32_t tmem = misc[0];

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const int row0 = s + kRows * m;
      mbar_arrive_expect_tx(bar(B_QFULL), kTile);
      tma_load_3d(sbase + kOffQ, &tm_q, bar(B_QFULL), 0, h, row0);
      tma_load_3d(sbase + kOffQ + kHalf, &tm_q, bar(B_QFULL), 64, h, row0);
      // K runs one tile ahead of V: K(n+1) is requested before V(n), whose
      // stage frees only when P(n-2).V completes.
      int k_last[kKStages] = {-1, -1, -1}, v_last[kVStages] = {-1, -1};
      bool ok = true;
      auto load_k = [&](int n) -> bool {
        const int st = n % kKStages, use = n / kKStages;
        if (use > 0 && !mbar_wait(bar(B_KEMPTY + st), (use - 1) & 1, abort_flag)) return false;
        const int krow = s + kCols * n;
        mbar_arrive_expect_tx(bar(B_KFULL + st), kTile);
        tma_load_3d(sbase + kOffK + st * kTile, &tm_k, bar(B_KFULL + st), 0, h, krow);
        tma_load_3d(sbase + kOffK + st * kTile + kHalf, &tm_k, bar(B_KFULL + st), 64, h, krow);
        k_last[st] = use;
        return true;
      };
      auto load_v = [&](int n) -> bool {
        const int st = n % kVStages, use = n / kVStages;
        if (use > 0 && !mbar_wait(bar(B_VEMPTY + st), (use - 1) & 1, abort_flag)) return false;
        const int krow = s + kCols * n;
        mbar_arrive_expect_tx(bar(B_VFULL + st), kTile);
        tma_load_3d(sbase + kOffV + st * kTile, &tm_v, bar(B_VFULL + st), 0, h, krow);
        tma_load_3d(sbase + kOffV + st * kTile + kHalf, &tm_v, bar(B_VFULL + st), 64, h, krow);
        v_last[st] = use;
        return true;
      };
      ok = load_k(0);
      for (int n = 0; n < nt && ok; ++n) {
        if (n + 1 < nt) ok = load_k(n + 1);
        if (ok) ok = load_v(n);
      }
      if (!ok) {
        set_status(a.status, kStatusTimeout);
        *abort_flag = 1;
        // Let the copies already issued land before shared memory goes away.
        mbar_wait(bar(B_QFULL), 0, nullptr);
        for (int st = 0; st < kKStages; ++st)
          if (k_last[st] >= 0) mbar_wait(bar(B_KFULL + st), k_last[st] & 1, nullptr);
        for (int st = 0; st < kVStages; ++st)
          if (v_last[st] >= 0) mbar_wait(bar(B_VFULL + st), v_last[st] & 1, nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(bar(B_QFULL), 0, abort_flag);
      auto issue_s = [&](int n) -> bool {
        const int st = n % kKStages;
        if (!mbar_wait(bar(B_KFULL + st), (n / kKStages) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t d = tmem + kColS0 + 128u * (n & 1);
        const uint32_t qa = sbase + kOffQ, ka = sbase + kOffK + st * kTile;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t off = (ks >> 2) * kHalf + (ks & 3) * 32;
          mma_ss(d, sw128_desc(qa + off, 16, 1024), sw128_desc(ka + off, 16, 1024), kIdescS,
                 ks > 0);
        }
        mma_commit(bar(B_KEMPTY + st));
        mma_commit(bar(B_SFULL + (n & 1)));
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok && nt > 1) ok = issue_s(1);
      for (int n = 0; n < nt && ok; ++n) {
        const int x = n & 1, st = n % kVStages;
        ok = mbar_wait(bar(B_PFULL + x), (n >> 1) & 1, abort_flag);
        if (!ok) break;
        ok = mbar_wait(bar(B_VFULL + st), (n / kVStages) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t va = sbase + kOffV + st * kTile;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          // 16 keys per step: rows 16ks.. of the V tile; the two 64-column
          // halves of d_v are 16 KB apart (leading byte offset).
          mma_ts(tmem + kColO, tmem + kColP0 + 64u * x + 8u * ks,
                 sw128_desc(va + ks * 2048, kHalf, 1024), kIdescPV, (n > 0 || ks > 0));
        }
        mma_commit(bar(B_VEMPTY + st));
        if (n + 2 < nt) ok = issue_s(n + 2);
      }
      if (!ok) {
        set_status(a.status, kStatusTimeout);
        *abort_flag = 1;
      }
      mma_commit(bar(B_OFULL));   // also marks every issued MMA as finished
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q4 = warp & 3;                      // TMEM lane quarter
    const int cq = (warp - 2) >> 2;               // column quarter of the S/O tiles
    const int r = q4 * 32 + lane;                 // row within the tile
    const int et = threadIdx.x - 64;              // 0..511 among epilogue threads
    const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
    const int i_loc = kRows * m + r;              // local row index in the sequence
    const bool row_ok = i_loc < n_b;
    const int t_row = s + (row_ok ? i_loc : 0);
    const float nrm = a.norm_len > 0 ? static_cast<float>(a.norm_len) : static_cast<float>(n_b);
    const int Lw = 2 * a.L - 1;
    uint8_t* wstage = smem + kOffWarp + (warp - 2) * kWarpStage;
    float* wv = reinterpret_cast<float*>(wstage);
    long long* wts = reinterpret_cast<long long*>(wstage + 96 * 4);
    const int team = (warp - 2) >> 3;             // S buffer / tile parity of this warp
    const int ch = ((warp - 2) >> 2) & 1;         // column half within the team's tiles
    EpiCtx ec;
    ec.thr = s_thr;
    ec.first = s_first;
    ec.rabt = s_rabt;
    ec.my_ts = TIME ? a.timestamps[t_row] : 0;
    ec.inv_n = 1.0f / nrm;
    ec.r = r;
    ec.lane = lane;
    bool ok = true;

    // Staging of this warp's 32 x 64 block of tile n: half position bias of
    // the 95 diagonals d = r - c in [32 q4 - 64 ch - 63, 32 q4 - 64 ch + 31]
    // (table index 128 (m - n) + d + L - 1), and the timestamps of its 64 keys
    // (keys past the sequence end repeat its last timestamp, which keeps them
    // non-decreasing; those keys are masked anyway).
    const int dbase = 32 * q4 - 64 * ch - 63;
    float pre_w0 = 0.f, pre_w1 = 0.f, pre_w2 = 0.f;
    long long pre_t0 = 0, pre_t1 = 0;
    auto prefetch = [&](int n) {
      if (POS) {
        const int t0 = kRows * (m - n) + dbase + lane + a.L - 1;
        const float* tab = a.rab_pos + static_cast<size_t>(h) * Lw;
        pre_w0 = (t0 >= 0 && t0 < Lw) ? __ldg(tab + t0) : 0.f;
        pre_w1 = (t0 + 32 >= 0 && t0 + 32 < Lw) ? __ldg(tab + t0 + 32) : 0.f;
        pre_w2 = (lane < 31 && t0 + 64 >= 0 && t0 + 64 < Lw) ? __ldg(tab + t0 + 64) : 0.f;
      }
      if (TIME) {
        const int j = kCols * n + 64 * ch + lane;
        pre_t0 = a.timestamps[s + (j < n_b ? j : n_b - 1)];
        pre_t1 = a.timestamps[s + (j + 32 < n_b ? j + 32 : n_b - 1)];
      }
    };
    bool sorted0 = true, sorted1 = true;
    auto stage = [&]() {   // previous users of the buffer (this warp) are done
      if (POS) {
        wv[lane] = 0.5f * pre_w0;
        wv[32 + lane] = 0.5f * pre_w1;
        wv[64 + lane] = 0.5f * pre_w2;
      }
      if (TIME) {
        wts[lane] = pre_t0;
        wts[32 + lane] = pre_t1;
        const long long n0 = __shfl_down_sync(0xffffffffu, pre_t0, 1);
        const long long n1 = __shfl_down_sync(0xffffffffu, pre_t1, 1);
        sorted0 = !__any_sync(0xffffffffu, lane < 31 && n0 < pre_t0);
        sorted1 = !__any_sync(0xffffffffu, lane < 31 && n1 < pre_t1);
      }
      __syncwarp();
    };
    if (team < nt) {
      prefetch(team);
      stage();
    }

    for (int n = team; n < nt; n += 2) {
      if (n + 2 < nt) prefetch(n + 2);            // global loads overlap this tile
      if (ok) ok = mbar_wait(bar(B_SFULL + team), (n >> 1) & 1, abort_flag);
      // The TMEM loads/stores below are warp-collective: keep the decision warp-uniform.
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t s_addr = tmem + lane_addr + kColS0 + 128u * team;
      const uint32_t p_addr = tmem + lane_addr + kColP0 + 64u * team;
      if (n == m)
        tile_to_p<POS, TIME, true>(s_addr, p_addr, 64 * ch, ec, wv, wts, sorted0, sorted1);
      else
        tile_to_p<POS, TIME, false>(s_addr, p_addr, 64 * ch, ec, wv, wts, sorted0, sorted1);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(B_PFULL + team));
      if (n + 2 < nt) stage();
    }

    // ---------------------------------------------- LayerNorm over heads + gate
    if (ok) ok = mbar_wait(bar(B_OFULL), 0, abort_flag);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) {
      set_status(a.status, kStatusTimeout);
      *abort_flag = 1;
    }
    tc_fence_after();
    const int H = a.H;
    const int D = H * 128;
    float* loc0 = reinterpret_cast<float*>(smem + kOffRed);   // [4][128] local partials
    float* loc1 = loc0 + kColGroups * 128;
    float* red0 = loc1 + kColGroups * 128;                      // [8][128] cluster slots
    float* red1 = red0 + 8 * 128;
    const uint32_t o_addr = tmem + lane_addr + kColO + 32u * cq;
    // The row's 32 values of this head and column quarter stay in registers.
    float ov[32];
    {
      uint32_t o0[32];
      tmem_ld32_nowait(o_addr, o0);
      tmem_wait_ld_dep(o0);
      // O accumulated N * SiLU(.) / N terms: apply 1/N here, in fp32.
#pragma unroll
      for (int i = 0; i < 32; ++i) ov[i] = __uint_as_float(o0[i]) * ec.inv_n;
    }
    const uint32_t lnbytes = static_cast<uint32_t>(H * 128 * 4);
    // pass 1: row sums.  The four column groups add up in shared memory, then
    // one thread per row sends this head's sum to every CTA of the cluster.
    float part = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) part += ov[i];
    loc0[cq * 128 + r] = part;
    named_bar_sync(1, kEpiThreads);
    if (cq == 0) {
      const float hsum = loc0[r] + loc0[128 + r] + loc0[256 + r] + loc0[384 + r];
      const uint32_t slot = smem_u32(red0 + h * 128 + r);
      for (int pr = 0; pr < H; ++pr)
        st_async_f32(mapa_shared(slot, pr), hsum, mapa_shared(bar_red0, pr));
    }
    if (et == 0) mbar_arrive_expect_tx(bar_red0, lnbytes);
    if (!mbar_wait<true>(bar_red0, 0, nullptr)) set_status(a.status, kStatusTimeout);
    float tot = 0.f;
    for (int k = 0; k < H; ++k) tot += red0[k * 128 + r];
    const float mean = tot / static_cast<float>(D);
    // pass 2: centred sum of squares, same route
    float sq = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float d0 = ov[i] - mean;
      sq = fmaf(d0, d0, sq);
    }
    loc1[cq * 128 + r] = sq;
    named_bar_sync(1, kEpiThreads);
    if (cq == 0) {
      const float hsq = loc1[r] + loc1[128 + r] + loc1[256 + r] + loc1[384 + r];
      const uint32_t slot = smem_u32(red1 + h * 128 + r);
      for (int pr = 0; pr < H; ++pr)
        st_async_f32(mapa_shared(slot, pr), hsq, mapa_shared(bar_red1, pr));
    }
    if (et == 0) mbar_arrive_expect_tx(bar_red1, lnbytes);
    if (!mbar_wait<true>(bar_red1, 0, nullptr)) set_status(a.status, kStatusTimeout);
    float totsq = 0.f;
    for (int k = 0; k < H; ++k) totsq += red1[k * 128 + r];
    const float var = totsq / static_cast<float>(D);
    const float rstd = 1.0f / sqrtf(var + a.eps);
    // pass 3: normalise, gate, store this thread's 32 columns
    if (row_ok) {
      const size_t rowD = static_cast<size_t>(t_row) * D + static_cast<size_t>(h) * 128 + 32 * cq;
      if (a.o_save) {
        float4* od = reinterpret_cast<float4*>(a.o_save + rowD);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          od[i] = make_float4(ov[4 * i], ov[4 * i + 1], ov[4 * i + 2], ov[4 * i + 3]);
      }
      const uint4* us = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(a.u) + rowD);
      uint4* yd = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.y) + rowD);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint4 uu = __ldg(us + i);
        const __nv_bfloat162* u2 = reinterpret_cast<const __nv_bfloat162*>(&uu);
        uint4 out;
        uint32_t* o32 = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 uf = __bfloat1622float2(u2[j]);
          const float y0 = (ov[8 * i + 2 * j] - mean) * rstd * silu_precise(uf.x);
          const float y1 = (ov[8 * i + 2 * j + 1] - mean) * rstd * silu_precise(uf.y);
          __nv_bfloat162 pr = __floats2bfloat162_rn(y0, y1);
          o32[j] = *reinterpret_cast<uint32_t*>(&pr);
        }
        yd[i] = out;
      }
      if (h == 0 && cq == 0 && a.ln_mean) {
        a.ln_mean[t_row] = mean;
        a.ln_rstd[t_row] = rstd;
      }
    }
    tc_fence_before();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    // Every MMA has completed once B_OFULL fired; wait for it before freeing TMEM.
    if (lane == 0) mbar_wait(bar(B_OFULL), 0, nullptr);
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <bool POS, bool TIME>
cudaError_t launch_variant(const FwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                           const CUtensorMap& tv, cudaStream_t stream) {
  // The shared-memory opt-in is a per-device function attribute: set it once
  // per device (not inside a stream capture of a later call).
  static bool configured[64] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    err = cudaFuncSetAttribute(hstu_fwd_bf16_sm100<POS, TIME>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return err;
    if (dev >= 0 && dev < 64) configured[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.H) * static_cast<unsigned>(a.B) *
                         static_cast<unsigned>(a.max_tiles),
                     1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(a.H);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, hstu_fwd_bf16_sm100<POS, TIME>, tq, tk, tv, a);
}

}  // namespace

cudaError_t launch_fwd_bf16_sm100(const FwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                                  const CUtensorMap& tv, cudaStream_t stream) {
  if (a.B == 0 || a.max_tiles == 0) return cudaSuccess;
  const bool pos = a.rab_pos != nullptr, tim = a.rab_time != nullptr;
  if (pos && tim) return launch_variant<true, true>(a, tq, tk, tv, stream);
  if (pos) return launch_variant<true, false>(a, tq, tk, tv, stream);
  if (tim) return launch_variant<false, true>(a, tq, tk, tv, stream);
  return launch_variant<false, false>(a, tq, tk, tv, stream);
}

}  // namespace hstu
