// plans.cu -- the shapes of the time-bias plans, computed once per call.
//
// The time bias of "HSTU Hierarchical Sequential Transduction Units" (§1 and
// §3: a per-head table indexed by the bucket of t_i - t_j) is applied by the
// attention kernels per warp and 32-column block through a plan (tile_math.cuh:
// the block's first bucket, up to three split columns, the kind).  A plan's
// shape depends on the timestamps only, not on the head, so this pass computes
// it once for every row and every block the row meets and the kernels of all
// H heads read it.  CTA (sequence b, row tile rt; group z of kPlanBlocks
// blocks); warp w takes rows 128 rt + 32 w + lane, the same 32-row groups as
// the kernels' epilogue warps, so the warp-level choice of kind is theirs.
#include "bounds.cuh"
#include "internal.h"
#include "tile_math.cuh"

namespace hstu {
namespace {

constexpr int kPlanThreads = 128;
constexpr int kPlanBlocks = 8;

struct PlanTab {
  const uint4* oct_;
  const unsigned* thr32_;
  __device__ __forceinline__ const uint4* oct() const { return oct_; }
  __device__ __forceinline__ const unsigned* thr32() const { return thr32_; }
};

// The extremes of a warp's 32 column timestamps (lane c holds column c's):
// the end lanes when they ascend, else a shuffle reduction.
__device__ __forceinline__ void block_range(long long kt, int lane, bool& asc, long long& lo,
                                            long long& hi) {
  const long long nx = __shfl_down_sync(0xffffffffu, kt, 1);
  asc = !__any_sync(0xffffffffu, lane < 31 && nx < kt);
  if (asc) {
    lo = __shfl_sync(0xffffffffu, kt, 0);
    hi = __shfl_sync(0xffffffffu, kt, 31);
  } else {
    lo = kt;
    hi = kt;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const long long x = __shfl_xor_sync(0xffffffffu, lo, o);
      const long long y = __shfl_xor_sync(0xffffffffu, hi, o);
      lo = x < lo ? x : lo;
      hi = y > hi ? y : hi;
    }
  }
}

__global__ void __launch_bounds__(kPlanThreads) time_plans(const __grid_constant__ PlanArgs a) {
  __shared__ uint4 s_oct[32];
  __shared__ unsigned s_thr32[kMaxBuckets];
  __shared__ uint32_t s_ts[kPlanThreads / 32][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned tiles = static_cast<unsigned>(a.max_tiles);
  const int rt = static_cast<int>(blockIdx.x % tiles), b = static_cast<int>(blockIdx.x / tiles);
  const int s = __ldg(a.offsets + b), e = __ldg(a.offsets + b + 1);
  const int n_b = e - s;
  const int jt = 4 * ((n_b + 127) / 128);             // blocks over the sequence's tiles
  const int j0 = static_cast<int>(blockIdx.y) * kPlanBlocks;
  // inconsistent offsets are reported by the attention kernels; groups of
  // blocks past the sequence, or (without the later-column plans) past the
  // row tile, have nothing to do (a uniform exit, before any barrier)
  if (s < 0 || n_b <= 0 || e > a.T || n_b > a.max_seq_len || 128 * rt >= n_b || j0 >= jt ||
      (!a.plan_up && j0 >= 4 * rt + 4))
    return;
  for (int i = threadIdx.x; i < 32; i += kPlanThreads) s_oct[i] = a.bt.oct[i];
  for (int i = threadIdx.x; i < kMaxBuckets; i += kPlanThreads) s_thr32[i] = a.bt.thr32[i];
  __syncthreads();
  const int i = 128 * rt + 32 * warp + lane;          // this thread's row of the sequence
  const bool row_ok = i < n_b;
  // rows past the end take the last row's timestamp, as in the kernels
  const long long my_ts =
      a.timestamps[checked(a.status, s + (row_ok ? i : n_b - 1), a.T, BS_BWD_TS)];
  const int j1 = min(jt, j0 + kPlanBlocks);
  const PlanTab tab{s_oct, s_thr32};
  uint32_t* ts32 = s_ts[warp];
  // the block's columns, those past the end repeating the last timestamp;
  // the next block's load is issued before this block's plans
  auto column_ts = [&](int jc) {
    const int j = 32 * jc + lane;
    return a.timestamps[checked(a.status, s + (j < n_b ? j : n_b - 1), a.T, BS_BWD_TS)];
  };
  long long kt_next = column_ts(j0);
  for (int jc = j0; jc < j1; ++jc) {
    const long long kt = kt_next;
    if (jc + 1 < j1) kt_next = column_ts(jc + 1);
    // columns at or before the row tile (dn); at or after it (up)
    const bool dn = a.plan_dn && jc < 4 * rt + 4, up = a.plan_up && jc >= 4 * rt;
    if (!dn && !up) continue;
    __syncwarp();
    ts32[lane] = static_cast<uint32_t>(kt);
    bool asc;
    long long lo, hi;
    block_range(kt, lane, asc, lo, hi);
    __syncwarp();
    const size_t at = static_cast<size_t>(jc) * a.T + s + (row_ok ? i : 0);
    // The block holding this warp's diagonal, the one before and (for the
    // rows-against-later-columns plans) the one after it: the bucket of every
    // element, for the per-element path (32-bit differences; the kernels use
    // these only where every |dt| of the block is below 2^31).
    const int jd = 4 * rt + warp;
    const int slot = jc == jd ? 0 : jc == jd - 1 ? 2 : (jc == jd + 1 && a.plan_up) ? 4 : -1;
    if (a.near && row_ok && slot >= 0) {
      const uint32_t my32 = static_cast<uint32_t>(my_ts);
      uint32_t w[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        uint32_t word = 0;
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
          const int d = static_cast<int>(my32 - ts32[4 * q + e2]);
          const int k = bucket32(static_cast<uint32_t>(d < 0 ? -d : d), tab.oct());
          word |= static_cast<uint32_t>(k) << (8 * e2);
        }
        w[q] = word;
      }
      uint4* dst = a.near + static_cast<size_t>(s + i) * 6 + slot;
      dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
      dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
    TimePlan p;
    if (dn) {
      const int tb = plan_shape_dn(p, my_ts, lo, hi, asc, ts32, tab);
      if (row_ok) a.plan_dn[at] = plan_word(p, tb);
    }
    if (up) {
      const int tb = plan_shape_up(p, my_ts, lo, hi, asc, ts32, tab);
      if (row_ok) a.plan_up[at] = plan_word(p, tb);
    }
  }
}

// Candidates against their user's history: CTA (micro-batch mt of 128
// candidates, user b, group z of kPlanBlocks history blocks); warp w takes
// candidates 128 mt + 32 w + lane, the same 32-row groups as the scoring
// kernel's epilogue warps.  Every candidate follows the whole history, so
// these are plans against earlier columns.
__global__ void __launch_bounds__(kPlanThreads) cand_plans(const __grid_constant__ CandArgs a) {
  __shared__ uint4 s_oct[32];
  __shared__ unsigned s_thr32[kMaxBuckets];
  __shared__ uint32_t s_ts[kPlanThreads / 32][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned tiles = static_cast<unsigned>(a.max_tiles);
  const int mt = static_cast<int>(blockIdx.x % tiles), b = static_cast<int>(blockIdx.x / tiles);
  const int c0 = __ldg(a.cand_offsets + b), cb = __ldg(a.cand_offsets + b + 1) - c0;
  const int s = __ldg(a.offsets + b), nb = __ldg(a.offsets + b + 1) - s;
  // inconsistent offsets are reported by the scoring kernel (a uniform exit,
  // before any barrier, as for groups of blocks past the history)
  if (c0 < 0 || cb <= 0 || c0 + cb > a.C || s < 0 || nb <= 0 || s + nb > a.T ||
      nb > a.max_seq_len || 128 * mt >= cb || 32 * static_cast<int>(blockIdx.y) * kPlanBlocks >= nb)
    return;
  for (int i = threadIdx.x; i < 32; i += kPlanThreads) s_oct[i] = a.bt.oct[i];
  for (int i = threadIdx.x; i < kMaxBuckets; i += kPlanThreads) s_thr32[i] = a.bt.thr32[i];
  __syncthreads();
  const int ci = 128 * mt + 32 * warp + lane;         // this thread's candidate of the user
  const bool row_ok = ci < cb;
  // candidates past the user's last take the first one's timestamp, as in the kernel
  const int cand = c0 + (row_ok ? ci : 0);
  const long long my_ts = a.cand_ts[checked(a.status, cand, a.C, BS_CAND_ROW)];
  const int jt = 4 * ((nb + 127) / 128);
  const int j0 = static_cast<int>(blockIdx.y) * kPlanBlocks;
  const int j1 = min(jt, j0 + kPlanBlocks);
  const PlanTab tab{s_oct, s_thr32};
  uint32_t* ts32 = s_ts[warp];
  auto column_ts = [&](int jc) {
    const int j = 32 * jc + lane;
    return a.timestamps[checked(a.status, s + (j < nb ? j : nb - 1), a.T, BS_CAND_TS)];
  };
  long long kt_next = column_ts(j0);
  for (int jc = j0; jc < j1; ++jc) {
    if (32 * jc >= nb) break;                          // blocks past the history are skipped
    const long long kt = kt_next;
    if (jc + 1 < j1 && 32 * (jc + 1) < nb) kt_next = column_ts(jc + 1);
    __syncwarp();
    ts32[lane] = static_cast<uint32_t>(kt);
    bool asc;
    long long lo, hi;
    block_range(kt, lane, asc, lo, hi);
    __syncwarp();
    TimePlan p;
    const int tb = plan_shape_dn(p, my_ts, lo, hi, asc, ts32, tab);
    if (row_ok) a.plan[static_cast<size_t>(jc) * a.C + cand] = plan_word(p, tb);
  }
}

}  // namespace

cudaError_t launch_cand_plans(const CandArgs& a, cudaStream_t stream) {
  if (a.B == 0 || a.max_tiles == 0 || !a.plan) return cudaSuccess;
  if (a.plan_j < 4 * ((a.max_seq_len + 127) / 128)) return cudaErrorInvalidValue;
  // (user, micro-batch) in x, the group of history blocks in y (y is limited
  // to 65535, x is not)
  const dim3 grid(static_cast<unsigned>(a.max_tiles) * static_cast<unsigned>(a.B),
                  (a.plan_j + kPlanBlocks - 1) / kPlanBlocks);
  if (grid.y > 65535u) return cudaErrorInvalidConfiguration;   // max_seq_len beyond 16.7M
  cand_plans<<<grid, kPlanThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_time_plans(const PlanArgs& a, cudaStream_t stream) {
  if (a.B == 0 || a.max_tiles == 0) return cudaSuccess;
  if (a.plan_j < 4 * a.max_tiles) return cudaErrorInvalidValue;
  // (sequence, row tile) in x, the group of column blocks in y
  const dim3 grid(static_cast<unsigned>(a.max_tiles) * static_cast<unsigned>(a.B),
                  (a.plan_j + kPlanBlocks - 1) / kPlanBlocks);
  if (grid.y > 65535u) return cudaErrorInvalidConfiguration;   // max_seq_len beyond 16.7M
  time_plans<<<grid, kPlanThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace hstu
