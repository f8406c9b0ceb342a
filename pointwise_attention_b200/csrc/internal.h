// internal.h -- declarations shared by the host API and the kernels of libhstu.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "hstu.h"

namespace hstu {

// Bits of the device status word (first 4 bytes of the workspace).
constexpr int kStatusBadOffsets = 1;   // offsets contradict T / max_seq_len / L
constexpr int kStatusTimeout = 2;      // a bounded wait ran out
constexpr int kStatusBounds = 4;       // an index check of the HSTU_DEBUG_BOUNDS build failed

// The 256-byte head of the workspace: word 0 is the status word; words 16 and
// 17 are the bf16 forward's work counter and finished-CTA counter.  The
// forward leaves both counters (and its per-item head counters) at zero when
// it ends, so a zero-filled workspace stays valid across calls.
constexpr int kSchedCounterWord = 16;
constexpr int kSchedDoneWord = 17;

constexpr int kMaxBuckets = 128;
// thr[k] = smallest |dt| with bucket(dt) >= k (thr[0] = 0); entries k >= NB
// hold INT64_MAX so the bucket search never passes NB-1.
constexpr int kThrLen = kMaxBuckets + 4;

struct BucketTable {
  long long thr[kThrLen];
  signed char first_k[64];   // bucket(2^e), e = 0..62
  // 32-bit form for |dt| < 2^31: thr32[k] = thr[k] (0xFFFFFFFF where thr[k]
  // >= 2^32 or k >= NB), and per octave e = 0..31 the packed
  // {bucket(2^e), thr32[k+1], thr32[k+2], thr32[k+3]} (at most three
  // thresholds lie in one octave, as ln 2 / 0.301 < 3).
  unsigned thr32[kMaxBuckets];
  uint4 oct[32];
};

// Arguments common to the forward kernels (bf16 tcgen05 and fp32 SIMT).
struct FwdArgs {
  const int32_t* offsets;
  const int64_t* timestamps;
  const float* rab_pos;
  const float* rab_time;
  const void* q;     // used by the SIMT path (the tcgen05 path reads q/k/v via TMA)
  const void* k;
  const void* v;
  const void* u;
  void* y;
  float* o_save;
  float* ln_mean;
  float* ln_rstd;
  int* status;
  int B, T, H, d_qk, d_v;
  int max_seq_len;
  int max_tiles;     // ceil(max_seq_len / 128)
  int L;             // rab_pos_len (0 if no position table)
  int nb;            // number of time buckets (0 if no time table)
  int norm_len;
  float eps;
  const float* ln_weight;   // [H*d_v] or nullptr (ones)
  const float* ln_bias;     // [H*d_v] or nullptr (zeros)
  int vec32;         // u, y and o_save (if given) are 32-byte aligned
  int group;         // bf16 forward: sequences per scheduling group (>= 1)
  // bf16 forward, workspace: per (sequence, query tile) count of heads done
  // [B * max_tiles], and per (token, head) row statistics of O
  // {mean, M2, shift, 0} [T * H] for the LayerNorm over heads.
  unsigned* item_cnt;
  float4* stats;
  // bf16 forward with a time table, workspace: the time-plan shapes of every
  // query row against every 32-key block, [4 * max_tiles][T] words, and the
  // per-element buckets of its blocks nearest the diagonal, [T][6] uint4
  const uint32_t* plan_dn;
  const uint4* near;
  BucketTable bt;
};

struct BwdArgs {
  const int32_t* offsets;
  const int64_t* timestamps;
  const float* rab_pos;
  const float* rab_time;
  const void* q;
  const void* k;
  const void* v;
  const void* u;
  const void* dy;
  const float* o_save;
  const float* ln_mean;
  const float* ln_rstd;
  void* dq;
  void* dk;
  void* dv;
  void* du;
  float* d_rab_pos;
  float* d_rab_time;
  const float* ln_weight;   // [H*d_v] or nullptr (ones)
  const float* ln_bias;     // [H*d_v] or nullptr (zeros)
  float* d_ln_weight;       // [H*d_v] or nullptr; zeroed by the caller of the kernels
  float* d_ln_bias;
  void* dO;          // workspace: dO in the compute dtype [T, H*d_v]
  // workspace (bf16 with timestamps): the time plans of every 32-row group and
  // 32-column block, [plan_j][T] words each: rows = queries against earlier
  // keys (dQ), rows = keys against later queries (dK, dV)
  uint32_t* plan_dn;
  uint32_t* plan_up;
  uint4* near;       // per-element buckets of the blocks nearest the diagonal, [T][6] uint4
  int plan_j;        // blocks per row: 4 * max_tiles
  int* status;
  int B, T, H, d_qk, d_v;
  int max_seq_len;
  int max_tiles;
  int L;
  int nb;
  int norm_len;
  float eps;
  BucketTable bt;
};

// Arguments of the time-plan pass: the shapes of the time-bias plans of every
// row against every 32-column block it meets (tile_math.cuh, plan_word),
// [plan_j][T] words each; plan_dn: rows against earlier columns (queries
// against keys), plan_up: rows against later columns (keys against queries),
// either may be null.
struct PlanArgs {
  const int32_t* offsets;
  const int64_t* timestamps;
  uint32_t* plan_dn;
  uint32_t* plan_up;
  // or null: per row, the buckets (one byte each) of the 32-column block that
  // holds its diagonal, of the block before and of the block after it:
  // [T][6] uint4, 32 bytes each
  uint4* near;
  int* status;
  int B, T, max_seq_len, max_tiles, plan_j;
  BucketTable bt;
};

// Arguments of the projection GEMMs (UVQK and output + residual + LayerNorm).
// A [rows, K] bf16 and B [N, K] bf16 are read through TMA maps; K % 64 == 0.
struct ProjArgs {
  const float* bias;        // [N] or nullptr
  const float* ln_weight;   // output projection: [E] or nullptr (ones)
  const float* ln_bias;     // output projection: [E] or nullptr (zeros)
  const void* res;          // output projection: residual X [T, E] bf16
  void* out0;               // UVQK: u [T, Nu]; output projection: z [T, E]
  void* out1;               // UVQK: v [T, Nu]
  void* out2;               // UVQK: q [T, Nq]
  void* out3;               // UVQK: k [T, Nq]
  float* mean;              // output projection: [T] or nullptr (with rstd)
  float* rstd;
  int* status;
  int T, K, E, Nu, Nq;
  int act;                  // UVQK: 1 = SiLU after the bias
  int vec32;                // every output pointer is 32-byte aligned
  float eps;
};

// Arguments of the candidate-scoring kernel (scoring against cached histories).
struct CandArgs {
  const int32_t* offsets;        // history [B+1]
  const int32_t* cand_offsets;   // candidates [B+1]
  const int64_t* timestamps;     // history [T] (with a time table)
  const int64_t* cand_ts;        // candidates [C] (with a time table)
  const float* rab_pos;          // [H, 2L-1] or nullptr
  const float* rab_time;         // [H, nb] or nullptr
  const void* q;                 // candidates [C, H, 128] bf16 (also read through TMA)
  const void* k;                 // candidates [C, H, 128]
  const void* v;                 // candidates [C, H, 128]
  const void* u;                 // candidates [C, H*128]
  void* y;                       // candidates [C, H*128]
  const float* ln_weight;        // [H*128] or nullptr
  const float* ln_bias;
  float* o_ws;                   // workspace: O / N per candidate [C, H*128] fp32
  unsigned* cnt;                 // workspace: head CTAs done per (user, micro-batch)
  // workspace (with a time table): the time-plan shape of every candidate
  // against every 32-event block of its user's history, [plan_j][C] words
  uint32_t* plan;
  int plan_j;
  // workspace or null: the users by history length, longest first (the CTA
  // order of the scoring grid); null: in index order
  int* order;
  int* status;
  int B, T, C, H;
  int max_tiles;                 // micro-batches per user in the grid
  int max_seq_len;
  int L, nb, norm_len;
  float eps;
  BucketTable bt;
};

// The synchronous argument checks of hstu_attn_bwd (all but the workspace's).
hstu_status_t check_bwd_args(const hstu_problem_t* p, const void* dy, const void* q,
                             const void* k, const void* v, const void* u, const float* o_save,
                             const float* ln_mean, const float* ln_rstd, const void* dq,
                             const void* dk, const void* dv, const void* du,
                             const float* d_rab_pos, const float* d_rab_time,
                             const float* d_ln_weight, const float* d_ln_bias);

// Kernel launchers (return cudaSuccess or the launch error).
cudaError_t launch_fwd_bf16_sm100(const FwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                                  const CUtensorMap& tv, cudaStream_t stream);
cudaError_t launch_fwd_f32_simt(const FwdArgs& a, cudaStream_t stream);
cudaError_t launch_bwd_f32_simt(const BwdArgs& a, cudaStream_t stream);
cudaError_t launch_bwd_bf16_simt(const BwdArgs& a, cudaStream_t stream);
cudaError_t launch_bwd_pre_bf16(const BwdArgs& a, cudaStream_t stream);
cudaError_t launch_cand_sm100(const CandArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                              const CUtensorMap& tv, cudaStream_t stream);
cudaError_t launch_uvqk_sm100(const ProjArgs& a, const CUtensorMap& tx, const CUtensorMap& tw,
                              cudaStream_t stream);
cudaError_t launch_out_sm100(const ProjArgs& a, const CUtensorMap& ty, const CUtensorMap& tw,
                             cudaStream_t stream);
cudaError_t launch_time_plans(const PlanArgs& a, cudaStream_t stream);
cudaError_t launch_cand_plans(const CandArgs& a, cudaStream_t stream);
cudaError_t launch_cand_order(const CandArgs& a, cudaStream_t stream);
cudaError_t launch_bwd_attn_bf16_sm100(const BwdArgs& a, const CUtensorMap* maps,
                                       cudaStream_t stream);

}  // namespace hstu
