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
// Roles (192 threads): warp 0 issues TMA, warp 1 allocates TMEM and issues the
// MMAs (one thread), warps 2..5 run the epilogue, one query row per thread
// (warp w reads TMEM lanes 32*(w%4) .. 32*(w%4)+31).
//
// TMEM (512 columns): S0 [0,128) S1 [128,256) O [256,384) P0 [384,448)
// P1 [448,512).  S = Q K^T is fp32; P = SiLU(S+bias)/N is packed bf16 pairs and
// is the A operand (from TMEM) of O += P V.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace hstu {
namespace {

constexpr int kThreads = 192;
constexpr int kRows = 128;                  // query rows per tile
constexpr int kCols = 128;                  // keys per tile
constexpr int kHalf = 16384;                // 128 rows x 64 bf16 (one 128B-swizzle slab)
constexpr int kTile = 2 * kHalf;            // 128 x 128 bf16
constexpr int kStages = 2;

// shared-memory map (byte offsets from a 1024-aligned base)
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kTile;                    // kStages tiles
constexpr int kOffV = kOffK + kStages * kTile;          // kStages tiles
constexpr int kOffWin = kOffV + kStages * kTile;        // 2 x 256 fp32 position-bias windows
constexpr int kOffKts = kOffWin + 2 * 256 * 4;          // 2 x 128 int64 key timestamps
constexpr int kOffThr = kOffKts + 2 * 128 * 8;          // kThrLen int64 thresholds
constexpr int kOffFirst = kOffThr + kThrLen * 8;        // 64 int8 first bucket per octave
constexpr int kOffRabT = kOffFirst + 64;                // 128 fp32 time-bias row
constexpr int kOffRed = kOffRabT + 128 * 4;             // 2 x 8 x 128 fp32 LN exchange
constexpr int kOffBar = kOffRed + 2 * 8 * 128 * 4;      // mbarriers (8 B each)
constexpr int kNumBars = 16;
constexpr int kOffMisc = kOffBar + kNumBars * 8;        // tmem base, abort flag
constexpr int kSmemBytes = kOffMisc + 64 + 1024;        // + alignment slack

// barrier indices
constexpr int B_QFULL = 0;
constexpr int B_KFULL = 1;    // +stage
constexpr int B_KEMPTY = 3;   // +stage
constexpr int B_VFULL = 5;    // +stage
constexpr int B_VEMPTY = 7;   // +stage
constexpr int B_SFULL = 9;    // +buffer
constexpr int B_PFULL = 11;   // +buffer
constexpr int B_PFREE = 13;   // +buffer
constexpr int B_OFULL = 15;
// the two LN exchange barriers live in the misc block
constexpr int kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColO = 256, kColP0 = 384;

constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false, false);   // Q (K-major) x K (K-major)
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, false, true);   // P (TMEM) x V (MN-major)

__device__ __forceinline__ void set_status(int* status, int bit) {
  if (status) atomicOr(status, bit);
}

// SiLU(x) / N = (x/2)(1 + tanh(x/2)) / N with one MUFU op (tanh.approx).
__device__ __forceinline__ float silu_scaled(float x, float half_inv_n) {
  float hx = 0.5f * x;
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(hx));
  float a = x * half_inv_n;
  return fmaf(a, t, a);
}

__device__ __forceinline__ float silu_precise(float x) { return x / (1.0f + __expf(-x)); }

// bucket(|dt|): start from the bucket of the octave's lower end, then pass at
// most three thresholds (ln 2 / 0.301 < 3 buckets per octave).
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
  if (s < 0 || n_b < 0 || e > a.T || n_b > a.max_seq_len || (a.rab_pos && n_b > a.L)) {
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
  const bool has_pos = a.rab_pos != nullptr;
  const bool has_time = a.rab_time != nullptr;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i)
      mbar_init(bar(i), (i == B_PFULL || i == B_PFULL + 1) ? 128u : 1u);
    mbar_init(bar_red0, 1);
    mbar_init(bar_red1, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sbase + kOffMisc, kTmemCols);
    tmem_relinquish();
  }
  if (warp >= 2 && has_time) {
    const int et = threadIdx.x - 64;
    for (int i = et; i < kThrLen; i += 128) s_thr[i] = a.bt.thr[i];
    if (et < 64) s_first[et] = a.bt.first_k[et];
    if (et < a.nb) s_rabt[et] = __ldg(a.rab_time + static_cast<size_t>(h) * a.nb + et);
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
      int last_use[kStages] = {-1, -1};
      bool ok = true;
      for (int n = 0; n < nt && ok; ++n) {
        const int st = n % kStages, use = n / kStages;
        const int krow = s + kCols * n;
        if (use > 0) ok = mbar_wait(bar(B_KEMPTY + st), (use - 1) & 1, abort_flag);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(B_KFULL + st), kTile);
        tma_load_3d(sbase + kOffK + st * kTile, &tm_k, bar(B_KFULL + st), 0, h, krow);
        tma_load_3d(sbase + kOffK + st * kTile + kHalf, &tm_k, bar(B_KFULL + st), 64, h, krow);
        if (use > 0) ok = mbar_wait(bar(B_VEMPTY + st), (use - 1) & 1, abort_flag);
        if (!ok) { last_use[st] = use; break; }
        mbar_arrive_expect_tx(bar(B_VFULL + st), kTile);
        tma_load_3d(sbase + kOffV + st * kTile, &tm_v, bar(B_VFULL + st), 0, h, krow);
        tma_load_3d(sbase + kOffV + st * kTile + kHalf, &tm_v, bar(B_VFULL + st), 64, h, krow);
        last_use[st] = use;
      }
      if (!ok) {
        set_status(a.status, kStatusTimeout);
        *abort_flag = 1;
        // Let the copies already issued land before shared memory goes away.
        mbar_wait(bar(B_QFULL), 0, nullptr);
        for (int st = 0; st < kStages; ++st)
          if (last_use[st] >= 0) {
            mbar_wait(bar(B_KFULL + st), last_use[st] & 1, nullptr);
            mbar_wait(bar(B_VFULL + st), last_use[st] & 1, nullptr);
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(bar(B_QFULL), 0, abort_flag);
      auto issue_s = [&](int n) -> bool {
        const int st = n % kStages;
        if (!mbar_wait(bar(B_KFULL + st), (n / kStages) & 1, abort_flag)) return false;
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
        const int x = n & 1, st = n % kStages;
        ok = mbar_wait(bar(B_PFULL + x), (n >> 1) & 1, abort_flag);
        if (!ok) break;
        ok = mbar_wait(bar(B_VFULL + st), (n / kStages) & 1, abort_flag);
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
        mma_commit(bar(B_PFREE + x));
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
    const int r = q4 * 32 + lane;                 // row within the tile
    const int et = threadIdx.x - 64;              // 0..127 among epilogue threads
    const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
    const int i_loc = kRows * m + r;              // local row index in the sequence
    const bool row_ok = i_loc < n_b;
    const int t_row = s + (row_ok ? i_loc : 0);
    const long long my_ts = has_time ? a.timestamps[t_row] : 0;
    const float nrm = a.norm_len > 0 ? static_cast<float>(a.norm_len) : static_cast<float>(n_b);
    const float half_inv_n = 0.5f / nrm;
    float* s_win = reinterpret_cast<float*>(smem + kOffWin);
    long long* s_kts = reinterpret_cast<long long*>(smem + kOffKts);
    const int Lw = 2 * a.L - 1;
    bool ok = true;

    // Every epilogue thread runs all nt iterations (work is skipped after a
    // failed wait) so the named barrier below always sees 128 threads.
    for (int n = 0; n < nt; ++n) {
      const int x = n & 1;
      float* win = s_win + 256 * x;
      long long* kts = s_kts + 128 * x;
      if (ok && has_pos) {
        // win[w] = rab_pos[h][(i - j) + L - 1] with i - j = 128 (m - n) + w - 127
        for (int w = et; w < 255; w += 128) {
          const int tbl = kRows * (m - n) + w - 127 + a.L - 1;
          win[w] = (tbl >= 0 && tbl < Lw) ? __ldg(a.rab_pos + static_cast<size_t>(h) * Lw + tbl)
                                          : 0.0f;
        }
      }
      if (ok && has_time) {
        const int j_loc = kCols * n + et;
        kts[et] = a.timestamps[s + (j_loc < n_b ? j_loc : 0)];
      }
      named_bar_sync(1, 128);
      if (ok) ok = mbar_wait(bar(B_SFULL + x), (n >> 1) & 1, abort_flag);
      if (ok && n >= 2) ok = mbar_wait(bar(B_PFREE + x), ((n - 2) >> 1) & 1, abort_flag);
      // The TMEM loads/stores below are warp-collective: keep the decision warp-uniform.
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) continue;
      tc_fence_after();
      const bool diag = (n == m);
      const uint32_t s_addr = tmem + lane_addr + kColS0 + 128u * x;
      const uint32_t p_addr = tmem + lane_addr + kColP0 + 64u * x;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        float v[32];
        tmem_ld32(s_addr + 32u * cc, v);
        tmem_wait_ld();
        uint32_t packed[16];
#pragma unroll
        for (int e2 = 0; e2 < 16; ++e2) {
          float y2[2];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int c = 32 * cc + 2 * e2 + hh;
            float sv = v[2 * e2 + hh];
            if (has_pos) sv += win[r - c + 127];
            if (has_time) sv += s_rabt[time_bucket(my_ts - kts[c], s_thr, s_first)];
            float yv = silu_scaled(sv, half_inv_n);
            if (diag && c > r) yv = 0.0f;
            y2[hh] = yv;
          }
          __nv_bfloat162 pr = __floats2bfloat162_rn(y2[0], y2[1]);
          packed[e2] = *reinterpret_cast<uint32_t*>(&pr);
        }
        tmem_st16(p_addr + 16u * cc, packed);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(B_PFULL + x));
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
    float* red0 = reinterpret_cast<float*>(smem + kOffRed);
    float* red1 = red0 + 8 * 128;
    const uint32_t o_addr = tmem + lane_addr + kColO;
    // pass 1: row sum of this head's 128 columns -> every CTA of the cluster
    float sum = 0.f;
    for (int cc = 0; cc < 4; ++cc) {
      float v[32];
      tmem_ld32(o_addr + 32u * cc, v);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; ++i) sum += v[i];
    }
    const uint32_t my_slot0 = smem_u32(red0 + h * 128 + r);
    for (int pr = 0; pr < H; ++pr)
      st_async_f32(mapa_shared(my_slot0, pr), sum, mapa_shared(bar_red0, pr));
    if (et == 0) mbar_arrive_expect_tx(bar_red0, static_cast<uint32_t>(H * 128 * 4));
    if (!mbar_wait<true>(bar_red0, 0, nullptr)) set_status(a.status, kStatusTimeout);
    float tot = 0.f;
    for (int hh = 0; hh < H; ++hh) tot += red0[hh * 128 + r];
    const float mean = tot / static_cast<float>(D);
    // pass 2: centred sum of squares
    float sq = 0.f;
    for (int cc = 0; cc < 4; ++cc) {
      float v[32];
      tmem_ld32(o_addr + 32u * cc, v);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float d0 = v[i] - mean;
        sq = fmaf(d0, d0, sq);
      }
    }
    const uint32_t my_slot1 = smem_u32(red1 + h * 128 + r);
    for (int pr = 0; pr < H; ++pr)
      st_async_f32(mapa_shared(my_slot1, pr), sq, mapa_shared(bar_red1, pr));
    if (et == 0) mbar_arrive_expect_tx(bar_red1, static_cast<uint32_t>(H * 128 * 4));
    if (!mbar_wait<true>(bar_red1, 0, nullptr)) set_status(a.status, kStatusTimeout);
    float totsq = 0.f;
    for (int hh = 0; hh < H; ++hh) totsq += red1[hh * 128 + r];
    const float var = totsq / static_cast<float>(D);
    const float rstd = 1.0f / sqrtf(var + a.eps);
    // pass 3: normalise, gate, store.  The TMEM loads are warp-collective, so
    // every lane issues them; only the global accesses depend on the row.
    const size_t rowD = static_cast<size_t>(t_row) * D + static_cast<size_t>(h) * 128;
    const __nv_bfloat16* urow = reinterpret_cast<const __nv_bfloat16*>(a.u) + rowD;
    __nv_bfloat16* yrow = reinterpret_cast<__nv_bfloat16*>(a.y) + rowD;
    for (int cc = 0; cc < 4; ++cc) {
      float v[32];
      tmem_ld32(o_addr + 32u * cc, v);
      tmem_wait_ld();
      if (!row_ok) continue;
      if (a.o_save) {
        float4* od = reinterpret_cast<float4*>(a.o_save + rowD + 32 * cc);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          od[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      }
      const uint4* us = reinterpret_cast<const uint4*>(urow + 32 * cc);
      uint4* yd = reinterpret_cast<uint4*>(yrow + 32 * cc);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint4 uu = __ldg(us + i);
        const __nv_bfloat162* u2 = reinterpret_cast<const __nv_bfloat162*>(&uu);
        uint4 out;
        uint32_t* o32 = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 uf = __bfloat1622float2(u2[j]);
          const float y0 = (v[8 * i + 2 * j] - mean) * rstd * silu_precise(uf.x);
          const float y1 = (v[8 * i + 2 * j + 1] - mean) * rstd * silu_precise(uf.y);
          __nv_bfloat162 pr = __floats2bfloat162_rn(y0, y1);
          o32[j] = *reinterpret_cast<uint32_t*>(&pr);
        }
        yd[i] = out;
      }
    }
    if (row_ok) {
      if (h == 0 && a.ln_mean) {
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

}  // namespace

cudaError_t launch_fwd_bf16_sm100(const FwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                                  const CUtensorMap& tv, cudaStream_t stream) {
  if (a.B == 0 || a.max_tiles == 0) return cudaSuccess;
  // The shared-memory opt-in is a per-device function attribute: set it once
  // per device (not inside a stream capture of a later call).
  static bool configured[64] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    err = cudaFuncSetAttribute(hstu_fwd_bf16_sm100, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kSmemBytes);
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
  return cudaLaunchKernelEx(&cfg, hstu_fwd_bf16_sm100, tq, tk, tv, a);
}

}  // namespace hstu
