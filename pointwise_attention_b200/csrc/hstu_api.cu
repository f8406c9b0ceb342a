// hstu_api.cu -- the C ABI of libhstu (declared in include/hstu.h): argument
// validation, workspace layout, the time-bucket threshold table, TMA tensor
// maps, and kernel dispatch.  No exception crosses the boundary.
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "hstu.h"
#include "internal.h"

using namespace hstu;

namespace {

// NVTX range around one library call (visible in Nsight timelines; a no-op
// unless a profiler injects its NVTX handler).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

constexpr size_t kAlign = 256;
constexpr size_t kStatusBytes = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------- time buckets
// bucket(a) for a >= 1 without the cap: floor(ln(a) / 0.301) in fp64.
int bucket_uncapped(long long a) {
  double x = static_cast<double>(a);
  if (x < 1.0) x = 1.0;
  return static_cast<int>(std::floor(std::log(x) / 0.301));
}

// thr_all[k] = smallest a >= 1 with bucket_uncapped(a) >= k, k = 1..127, found by
// binary search (the bucket is non-decreasing in a).
struct Thresholds {
  long long thr[kMaxBuckets];
};

const Thresholds& thresholds() {
  static Thresholds t;
  static std::once_flag once;
  std::call_once(once, [] {
    t.thr[0] = 0;
    for (int k = 1; k < kMaxBuckets; ++k) {
      long long lo = 1, hi = 0x7FFFFFFFFFFFFFFFll;
      while (lo < hi) {
        const long long mid = lo + (hi - lo) / 2;
        if (bucket_uncapped(mid) >= k) hi = mid; else lo = mid + 1;
      }
      t.thr[k] = lo;
    }
  });
  return t;
}

void fill_bucket_table(BucketTable* bt, int nb) {
  const Thresholds& t = thresholds();
  for (int k = 0; k < kThrLen; ++k)
    bt->thr[k] = (k < nb && k < kMaxBuckets) ? t.thr[k] : 0x7FFFFFFFFFFFFFFFll;
  for (int e = 0; e < 64; ++e) {
    const long long p = (e < 63) ? (1ll << e) : 0x7FFFFFFFFFFFFFFFll;
    int k = 0;
    while (k + 1 < nb && bt->thr[k + 1] <= p) ++k;
    bt->first_k[e] = static_cast<signed char>(k);
  }
  for (int k = 0; k < kMaxBuckets; ++k)
    bt->thr32[k] = (bt->thr[k] <= 0xFFFFFFFFll) ? static_cast<unsigned>(bt->thr[k]) : 0xFFFFFFFFu;
  for (int e = 0; e < 32; ++e) {
    const int k = bt->first_k[e];
    auto t = [&](int i) { return k + i < kMaxBuckets ? bt->thr32[k + i] : 0xFFFFFFFFu; };
    bt->oct[e] = make_uint4(static_cast<unsigned>(k), t(1), t(2), t(3));
  }
}

// ---------------------------------------------------------- TMA tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [T, H, 128] bf16 viewed as a 3-D tensor (d, head, token); box = 64 x 1 x 128,
// 128-byte swizzle: one box is one 128-row x 128-byte slab of a K-major tile.
bool make_map_3d(CUtensorMap* map, const void* base, int T, int H, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(T)};
  cuuint64_t strides[2] = {128 * 2, static_cast<cuuint64_t>(H) * 128 * 2};
  cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// [rows, cols] bf16 row-major as a 2-D tensor (col, row); box = 64 x box_rows,
// 128-byte swizzle: one box is box_rows rows x 128 bytes of a K-major tile.
// Rows past `rows` read as zeros.
bool make_map_2d(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------- validation
hstu_status_t check_problem(const hstu_problem_t* p) {
  if (!p) return HSTU_ERR_INVALID_ARG;
  if (p->dtype != HSTU_F32 && p->dtype != HSTU_BF16) return HSTU_ERR_INVALID_ARG;
  if (p->batch < 0 || p->total_tokens < 0 || p->max_seq_len < 0 || p->num_heads < 1 ||
      p->d_qk < 1 || p->d_v < 1 || p->norm_len < 0)
    return HSTU_ERR_INVALID_ARG;
  if (!(p->ln_eps > 0.0f) || !std::isfinite(p->ln_eps)) return HSTU_ERR_INVALID_ARG;
  if (p->batch > 0 && !p->offsets) return HSTU_ERR_INVALID_ARG;
  if (p->batch == 0 && p->total_tokens != 0) return HSTU_ERR_INVALID_ARG;
  if (p->rab_pos && (p->rab_pos_len < 1 || p->rab_pos_len < p->max_seq_len))
    return HSTU_ERR_INVALID_ARG;
  if (p->rab_pos && static_cast<int64_t>(p->rab_pos_len) * 2 - 1 > 0x7FFFFFFF)
    return HSTU_ERR_INVALID_ARG;
  if (p->rab_time && (!p->timestamps || p->num_time_buckets < 1 ||
                      p->num_time_buckets > kMaxBuckets))
    return HSTU_ERR_INVALID_ARG;
  if (p->offsets_host) {
    const int32_t* o = p->offsets_host;
    if (o[0] != 0 || o[p->batch] != p->total_tokens) return HSTU_ERR_INVALID_ARG;
    for (int b = 0; b < p->batch; ++b) {
      const int64_t n = static_cast<int64_t>(o[b + 1]) - o[b];
      if (n < 0 || n > p->max_seq_len) return HSTU_ERR_INVALID_ARG;
      if (p->rab_pos && n > p->rab_pos_len) return HSTU_ERR_INVALID_ARG;
    }
  }
  return HSTU_OK;
}

bool bf16_supported(const hstu_problem_t* p) {
  // The forward numbers its (sequence, query tile, head) work slots in 32
  // bits (with room for one scheduling group more and a claim window), and
  // the backward launches one CTA per (head, sequence, tile).
  const int64_t tiles = (p->max_seq_len + 127) / 128;
  const int64_t slots = 2 * static_cast<int64_t>(p->batch) * tiles * p->num_heads;
  return p->dtype == HSTU_BF16 && p->d_qk == 128 && p->d_v == 128 && p->num_heads <= 8 &&
         slots <= 0x7FFFFF00LL;
}

bool f32_supported(const hstu_problem_t* p) {
  return p->dtype == HSTU_F32 && p->d_qk <= 128 && p->d_v <= 128 &&
         p->num_heads * p->d_v <= 1024;
}

// Workspace layout:
//   forward (bf16): [status 256 B][per (sequence, query tile) head counters:
//                    B * ceil(max_seq_len/128) u32][per (token, head) row
//                    statistics: T * H float4] and, with a time table,
//                    [time plans (queries against keys): J * T u32]
//                    [the buckets of the blocks nearest the diagonal: T * 96 B]
//   backward:       [status 256 B][dO: T*H*dv in the input dtype]
//                    and, bf16 with a time table, [time plans: 2 * J * T u32]
//                    with J = 4 * ceil(max_seq_len / 128)
struct WsLayout {
  size_t cnt_off, stats_off, dO_off, plan_off, near_off, total;
  int plan_j;
};

WsLayout ws_layout(const hstu_problem_t* p, int is_bwd) {
  WsLayout l{};
  size_t off = kStatusBytes;
  const size_t T = static_cast<size_t>(p->total_tokens);
  if (is_bwd) {
    l.dO_off = off;
    off += align_up(T * p->num_heads * p->d_v * (p->dtype == HSTU_BF16 ? 2 : 4));
    if (p->dtype == HSTU_BF16 && p->rab_time) {
      l.plan_j = 4 * ((p->max_seq_len + 127) / 128);
      l.plan_off = off;
      off += align_up(2 * static_cast<size_t>(l.plan_j) * T * 4);
      l.near_off = off;
      off += align_up(T * 96);
    }
  } else if (p->dtype == HSTU_BF16) {
    const size_t tiles = static_cast<size_t>((p->max_seq_len + 127) / 128);
    l.cnt_off = off;
    off += align_up(static_cast<size_t>(p->batch) * tiles * 4);
    l.stats_off = off;
    off += align_up(T * p->num_heads * 16);
    if (p->rab_time) {
      l.plan_j = 4 * static_cast<int>(tiles);
      l.plan_off = off;
      off += align_up(static_cast<size_t>(l.plan_j) * T * 4);
      l.near_off = off;
      off += align_up(T * 96);
    }
  }
  l.total = off;
  return l;
}

hstu_status_t check_ws(const hstu_problem_t* p, int is_bwd, void* ws, size_t bytes) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0) return HSTU_ERR_WORKSPACE;
  if (bytes < ws_layout(p, is_bwd).total) return HSTU_ERR_WORKSPACE;
  return HSTU_OK;
}

void fill_common(const hstu_problem_t* p, int* status, FwdArgs* a) {
  a->offsets = p->offsets;
  a->timestamps = p->timestamps;
  a->rab_pos = p->rab_pos;
  a->rab_time = p->rab_time;
  a->status = status;
  a->B = p->batch;
  a->T = p->total_tokens;
  a->H = p->num_heads;
  a->d_qk = p->d_qk;
  a->d_v = p->d_v;
  a->max_seq_len = p->max_seq_len;
  a->max_tiles = (p->max_seq_len + 127) / 128;
  a->L = p->rab_pos ? p->rab_pos_len : 0;
  a->nb = p->rab_time ? p->num_time_buckets : 0;
  a->norm_len = p->norm_len;
  a->eps = p->ln_eps;
  a->ln_weight = p->ln_weight;
  a->ln_bias = p->ln_bias;
  fill_bucket_table(&a->bt, p->rab_time ? p->num_time_buckets : 1);
}

}  // namespace

extern "C" {

size_t hstu_attn_workspace_size(const hstu_problem_t* p, int is_bwd) {
  if (check_problem(p) != HSTU_OK) return 0;
  return ws_layout(p, is_bwd ? 1 : 0).total;
}

const char* hstu_status_string(hstu_status_t s) {
  switch (s) {
    case HSTU_OK: return "HSTU_OK";
    case HSTU_ERR_INVALID_ARG: return "HSTU_ERR_INVALID_ARG: invalid argument";
    case HSTU_ERR_UNSUPPORTED: return "HSTU_ERR_UNSUPPORTED: shape or dtype not implemented";
    case HSTU_ERR_CUDA: return "HSTU_ERR_CUDA: a CUDA call or launch failed";
    case HSTU_ERR_TIMEOUT: return "HSTU_ERR_TIMEOUT: a bounded device wait ran out";
    case HSTU_ERR_WORKSPACE: return "HSTU_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case HSTU_ERR_BOUNDS: return "HSTU_ERR_BOUNDS: a debug-build index check failed";
  }
  return "HSTU: unknown status";
}

int32_t hstu_time_bucket_thresholds(int64_t* out, int32_t num_buckets) {
  if (!out || num_buckets < 1 || num_buckets > kMaxBuckets) return -1;
  BucketTable bt;
  fill_bucket_table(&bt, num_buckets);
  for (int k = 1; k < num_buckets; ++k) out[k - 1] = bt.thr[k];
  return num_buckets - 1;
}

hstu_status_t hstu_attn_fwd(const hstu_problem_t* p, const void* q, const void* k, const void* v,
                            const void* u, void* y, float* o_save, float* ln_mean,
                            float* ln_rstd, void* workspace, size_t workspace_bytes,
                            void* stream) {
  NvtxRange range("hstu_attn_fwd");
  hstu_status_t st = check_problem(p);
  if (st != HSTU_OK) return st;
  if (p->total_tokens > 0) {
    if (!q || !k || !v || !u || !y) return HSTU_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(u) || !aligned16(y))
      return HSTU_ERR_INVALID_ARG;
  }
  const int nsave = (o_save != nullptr) + (ln_mean != nullptr) + (ln_rstd != nullptr);
  if (nsave != 0 && nsave != 3) return HSTU_ERR_INVALID_ARG;
  if (o_save && !aligned16(o_save)) return HSTU_ERR_INVALID_ARG;
  if (!bf16_supported(p) && !f32_supported(p)) return HSTU_ERR_UNSUPPORTED;
  st = check_ws(p, 0, workspace, workspace_bytes);
  if (st != HSTU_OK) return st;
  if (p->total_tokens == 0 || p->batch == 0) return HSTU_OK;

  FwdArgs a;
  std::memset(&a, 0, sizeof(a));
  fill_common(p, static_cast<int*>(workspace), &a);
  a.q = q; a.k = k; a.v = v; a.u = u; a.y = y;
  a.o_save = o_save; a.ln_mean = ln_mean; a.ln_rstd = ln_rstd;
  // Scheduling groups of the bf16 forward: as many sequences as keep their K
  // and V (at max_seq_len) within about 40 MB of the 126 MB L2.
  {
    const double kv = static_cast<double>(p->max_seq_len) * p->num_heads *
                      (p->d_qk + p->d_v) * 2.0;
    const double g = kv > 0 ? std::floor(40.0e6 / kv) : p->batch;
    a.group = static_cast<int>(std::max(1.0, std::min(static_cast<double>(p->batch), g)));
  }
  auto al32 = [](const void* x) { return (reinterpret_cast<uintptr_t>(x) & 31u) == 0; };
  a.vec32 = al32(u) && al32(y) && (!o_save || al32(o_save));
  const WsLayout l = ws_layout(p, 0);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.item_cnt = reinterpret_cast<unsigned*>(ws + l.cnt_off);
  a.stats = reinterpret_cast<float4*>(ws + l.stats_off);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t err = cudaSuccess;
  if (p->dtype == HSTU_BF16) {
    CUtensorMap tq, tk, tv;
    if (!make_map_3d(&tq, q, p->total_tokens, p->num_heads, 128) ||
        !make_map_3d(&tk, k, p->total_tokens, p->num_heads, 128) ||
        !make_map_3d(&tv, v, p->total_tokens, p->num_heads, 128))
      return HSTU_ERR_CUDA;
    if (l.plan_j > 0) {
      // the time-plan shapes, once for all heads
      uint32_t* plans = reinterpret_cast<uint32_t*>(ws + l.plan_off);
      a.plan_dn = plans;
      a.near = reinterpret_cast<const uint4*>(ws + l.near_off);
      PlanArgs pa;
      std::memset(&pa, 0, sizeof(pa));
      pa.offsets = a.offsets;
      pa.timestamps = a.timestamps;
      pa.plan_dn = plans;
      pa.near = reinterpret_cast<uint4*>(ws + l.near_off);
      pa.status = a.status;
      pa.B = a.B;
      pa.T = a.T;
      pa.max_seq_len = a.max_seq_len;
      pa.max_tiles = a.max_tiles;
      pa.plan_j = l.plan_j;
      pa.bt = a.bt;
      err = launch_time_plans(pa, s);
    }
    if (err == cudaSuccess) err = launch_fwd_bf16_sm100(a, tq, tk, tv, s);
  } else {
    err = launch_fwd_f32_simt(a, s);
  }
  return err == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

}  // extern "C"

// Every check hstu_attn_bwd makes before it enqueues anything, except the
// workspace's (shared with the workspace-free entry point).
hstu_status_t hstu::check_bwd_args(const hstu_problem_t* p, const void* dy, const void* q,
                                   const void* k, const void* v, const void* u,
                                   const float* o_save, const float* ln_mean,
                                   const float* ln_rstd, const void* dq, const void* dk,
                                   const void* dv, const void* du, const float* d_rab_pos,
                                   const float* d_rab_time, const float* d_ln_weight,
                                   const float* d_ln_bias) {
  hstu_status_t st = check_problem(p);
  if (st != HSTU_OK) return st;
  if (p->total_tokens > 0) {
    const void* ptrs[] = {dy, q, k, v, u, o_save, ln_mean, ln_rstd, dq, dk, dv, du};
    for (const void* x : ptrs)
      if (!x) return HSTU_ERR_INVALID_ARG;
    const void* al[] = {dy, q, k, v, u, o_save, dq, dk, dv, du};
    for (const void* x : al)
      if (!aligned16(x)) return HSTU_ERR_INVALID_ARG;
  }
  if (d_rab_pos && !p->rab_pos) return HSTU_ERR_INVALID_ARG;
  if (d_rab_time && !p->rab_time) return HSTU_ERR_INVALID_ARG;
  if (d_ln_weight && !p->ln_weight) return HSTU_ERR_INVALID_ARG;
  if (d_ln_bias && !p->ln_bias) return HSTU_ERR_INVALID_ARG;
  if (!bf16_supported(p) && !f32_supported(p)) return HSTU_ERR_UNSUPPORTED;
  return HSTU_OK;
}

extern "C" {

hstu_status_t hstu_attn_bwd(const hstu_problem_t* p, const void* dy, const void* q, const void* k,
                            const void* v, const void* u, const float* o_save,
                            const float* ln_mean, const float* ln_rstd, void* dq, void* dk,
                            void* dv, void* du, float* d_rab_pos, float* d_rab_time,
                            float* d_ln_weight, float* d_ln_bias, void* workspace,
                            size_t workspace_bytes, void* stream) {
  NvtxRange range("hstu_attn_bwd");
  hstu_status_t st = check_bwd_args(p, dy, q, k, v, u, o_save, ln_mean, ln_rstd, dq, dk, dv, du,
                                    d_rab_pos, d_rab_time, d_ln_weight, d_ln_bias);
  if (st != HSTU_OK) return st;
  st = check_ws(p, 1, workspace, workspace_bytes);
  if (st != HSTU_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d_rab_pos &&
      cudaMemsetAsync(d_rab_pos, 0,
                      sizeof(float) * p->num_heads * (2 * static_cast<size_t>(p->rab_pos_len) - 1),
                      s) != cudaSuccess)
    return HSTU_ERR_CUDA;
  if (d_rab_time &&
      cudaMemsetAsync(d_rab_time, 0, sizeof(float) * p->num_heads * p->num_time_buckets, s) !=
          cudaSuccess)
    return HSTU_ERR_CUDA;
  const size_t Dbytes = sizeof(float) * p->num_heads * p->d_v;
  if (d_ln_weight && cudaMemsetAsync(d_ln_weight, 0, Dbytes, s) != cudaSuccess) return HSTU_ERR_CUDA;
  if (d_ln_bias && cudaMemsetAsync(d_ln_bias, 0, Dbytes, s) != cudaSuccess) return HSTU_ERR_CUDA;
  if (p->total_tokens == 0 || p->batch == 0) return HSTU_OK;

  const WsLayout l = ws_layout(p, 1);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  FwdArgs common;
  std::memset(&common, 0, sizeof(common));
  fill_common(p, reinterpret_cast<int*>(ws), &common);
  BwdArgs a;
  std::memset(&a, 0, sizeof(a));
  a.offsets = common.offsets; a.timestamps = common.timestamps;
  a.rab_pos = common.rab_pos; a.rab_time = common.rab_time;
  a.q = q; a.k = k; a.v = v; a.u = u; a.dy = dy;
  a.o_save = o_save; a.ln_mean = ln_mean; a.ln_rstd = ln_rstd;
  a.dq = dq; a.dk = dk; a.dv = dv; a.du = du;
  a.d_rab_pos = d_rab_pos; a.d_rab_time = d_rab_time;
  a.ln_weight = p->ln_weight; a.ln_bias = p->ln_bias;
  a.d_ln_weight = d_ln_weight; a.d_ln_bias = d_ln_bias;
  a.dO = ws + l.dO_off;
  if (l.plan_j > 0) {
    a.plan_j = l.plan_j;
    a.plan_dn = reinterpret_cast<uint32_t*>(ws + l.plan_off);
    a.plan_up = a.plan_dn + static_cast<size_t>(l.plan_j) * p->total_tokens;
    a.near = reinterpret_cast<uint4*>(ws + l.near_off);
  }
  a.status = common.status;
  a.B = common.B; a.T = common.T; a.H = common.H; a.d_qk = common.d_qk; a.d_v = common.d_v;
  a.max_seq_len = common.max_seq_len; a.max_tiles = common.max_tiles;
  a.L = common.L; a.nb = common.nb; a.norm_len = common.norm_len; a.eps = common.eps;
  a.bt = common.bt;
  cudaError_t err;
  if (p->dtype == HSTU_BF16) {
    // q, k, v, dO with 128-row boxes (resident tiles), then 64-row boxes
    // (the sub-tile rings)
    CUtensorMap maps[8];
    const void* src[4] = {q, k, v, a.dO};
    for (int i = 0; i < 8; ++i)
      if (!make_map_3d(&maps[i], src[i & 3], p->total_tokens, p->num_heads, i < 4 ? 128 : 64))
        return HSTU_ERR_CUDA;
    err = launch_bwd_pre_bf16(a, s);                       // dU and dO (LayerNorm + gate)
    if (err == cudaSuccess) err = launch_bwd_attn_bf16_sm100(a, maps, s);   // dQ, dK, dV, d_rab
  } else {
    err = launch_bwd_f32_simt(a, s);
  }
  return err == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

hstu_status_t hstu_attn_check(void* workspace, void* stream) {
  if (!workspace) return HSTU_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return HSTU_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return HSTU_ERR_CUDA;
  if (word != 0) {
    if (cudaMemsetAsync(workspace, 0, sizeof(int), s) != cudaSuccess) return HSTU_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return HSTU_ERR_CUDA;
  }
  if (word & kStatusTimeout) return HSTU_ERR_TIMEOUT;
  if (word & kStatusBadOffsets) return HSTU_ERR_INVALID_ARG;
  if (word & kStatusBounds) return HSTU_ERR_BOUNDS;
  return HSTU_OK;
}

// ---------------------------------------------------------- projections
static bool al32(const void* x) { return (reinterpret_cast<uintptr_t>(x) & 31u) == 0; }

static hstu_status_t check_status_ws(void* ws, size_t bytes) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0 || bytes < kStatusBytes)
    return HSTU_ERR_WORKSPACE;
  return HSTU_OK;
}

hstu_status_t hstu_uvqk_fwd(int32_t T, int32_t E, int32_t H, int32_t d_qk, int32_t d_v,
                            int32_t act, const void* x, const void* w, const float* bias, void* u,
                            void* v, void* q, void* k, void* workspace, size_t workspace_bytes,
                            void* stream) {
  NvtxRange range("hstu_uvqk_fwd");
  if (T < 0 || E < 1 || H < 1 || d_qk < 1 || d_v < 1 || (act != 0 && act != 1))
    return HSTU_ERR_INVALID_ARG;
  const void* ptrs[] = {x, w, u, v, q, k};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return HSTU_ERR_INVALID_ARG;
  if (bias && !aligned16(bias)) return HSTU_ERR_INVALID_ARG;
  const int64_t Nu = static_cast<int64_t>(H) * d_v, Nq = static_cast<int64_t>(H) * d_qk;
  if (E % 64 != 0 || Nu % 256 != 0 || Nq % 256 != 0 || 2 * (Nu + Nq) > 65535 * 256 ||
      (static_cast<int64_t>(T) + 127) / 128 > 65535)
    return HSTU_ERR_UNSUPPORTED;
  hstu_status_t st = check_status_ws(workspace, workspace_bytes);
  if (st != HSTU_OK) return st;
  if (T == 0) return HSTU_OK;
  ProjArgs a;
  std::memset(&a, 0, sizeof(a));
  a.bias = bias;
  a.out0 = u; a.out1 = v; a.out2 = q; a.out3 = k;
  a.status = static_cast<int*>(workspace);
  a.T = T; a.K = E; a.E = E;
  a.Nu = static_cast<int>(Nu); a.Nq = static_cast<int>(Nq);
  a.act = act;
  a.vec32 = al32(u) && al32(v) && al32(q) && al32(k);
  CUtensorMap tx, tw;
  if (!make_map_2d(&tx, x, T, E, 128) || !make_map_2d(&tw, w, 2 * (Nu + Nq), E, 256))
    return HSTU_ERR_CUDA;
  const cudaError_t err = launch_uvqk_sm100(a, tx, tw, static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

hstu_status_t hstu_out_fwd(int32_t T, int32_t E, int32_t D, const void* y, const void* w,
                           const void* x, const float* bias, const float* ln_weight,
                           const float* ln_bias, float eps, void* z, float* mean, float* rstd,
                           void* workspace, size_t workspace_bytes, void* stream) {
  NvtxRange range("hstu_out_fwd");
  if (T < 0 || E < 1 || D < 1 || !(eps > 0.0f) || !std::isfinite(eps)) return HSTU_ERR_INVALID_ARG;
  const void* ptrs[] = {y, w, x, z};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return HSTU_ERR_INVALID_ARG;
  const void* opt[] = {bias, ln_weight, ln_bias};
  for (const void* p : opt)
    if (p && !aligned16(p)) return HSTU_ERR_INVALID_ARG;
  if ((mean == nullptr) != (rstd == nullptr)) return HSTU_ERR_INVALID_ARG;
  if ((E != 256 && E != 512) || D % 64 != 0) return HSTU_ERR_UNSUPPORTED;
  hstu_status_t st = check_status_ws(workspace, workspace_bytes);
  if (st != HSTU_OK) return st;
  if (T == 0) return HSTU_OK;
  ProjArgs a;
  std::memset(&a, 0, sizeof(a));
  a.bias = bias;
  a.ln_weight = ln_weight;
  a.ln_bias = ln_bias;
  a.res = x;
  a.out0 = z;
  a.mean = mean;
  a.rstd = rstd;
  a.status = static_cast<int*>(workspace);
  a.T = T; a.K = D; a.E = E;
  a.eps = eps;
  a.vec32 = al32(z);
  CUtensorMap ty, tw;
  if (!make_map_2d(&ty, y, T, D, 128) || !make_map_2d(&tw, w, E, D, 256)) return HSTU_ERR_CUDA;
  const cudaError_t err = launch_out_sm100(a, ty, tw, static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

// ---------------------------------------------------------- candidate scoring
static size_t cand_tiles(int32_t max_cands) { return (static_cast<size_t>(max_cands) + 127) / 128; }

// Candidate workspace: [status][per (user, micro-batch) counters][O / N per
// candidate, fp32][with a time table: plan words, J * C u32 with
// J = 4 * ceil(max_seq_len / 128)][the users' CTA order, B int32, up to
// kCandOrderMax users]
constexpr int kCandOrderMax = 4096;
static size_t cand_plan_j(const hstu_problem_t* p) {
  return p->rab_time ? 4 * static_cast<size_t>((p->max_seq_len + 127) / 128) : 0;
}

size_t hstu_cand_workspace_size(const hstu_problem_t* p, int32_t total_cands, int32_t max_cands) {
  if (check_problem(p) != HSTU_OK || total_cands < 0 || max_cands < 0) return 0;
  return kStatusBytes + align_up(static_cast<size_t>(p->batch) * cand_tiles(max_cands) * 4) +
         align_up(static_cast<size_t>(total_cands) * p->num_heads * p->d_v * 4) +
         align_up(cand_plan_j(p) * static_cast<size_t>(total_cands) * 4) +
         (p->batch <= kCandOrderMax ? align_up(static_cast<size_t>(p->batch) * 4) : 0);
}

hstu_status_t hstu_cand_fwd(const hstu_problem_t* p, const void* k_hist, const void* v_hist,
                            const int32_t* cand_offsets, int32_t total_cands, int32_t max_cands,
                            const int64_t* cand_timestamps, const void* q, const void* k,
                            const void* v, const void* u, void* y, void* workspace,
                            size_t workspace_bytes, void* stream) {
  NvtxRange range("hstu_cand_fwd");
  hstu_status_t st = check_problem(p);
  if (st != HSTU_OK) return st;
  if (total_cands < 0 || max_cands < 0 || (total_cands > 0 && max_cands < 1))
    return HSTU_ERR_INVALID_ARG;
  if (p->batch > 0 && !cand_offsets) return HSTU_ERR_INVALID_ARG;
  if (p->rab_pos && p->rab_pos_len < p->max_seq_len + 1) return HSTU_ERR_INVALID_ARG;
  if (p->rab_time && total_cands > 0 && !cand_timestamps) return HSTU_ERR_INVALID_ARG;
  if (total_cands > 0) {
    const void* ptrs[] = {q, k, v, u, y};
    for (const void* x : ptrs)
      if (!x || !aligned16(x)) return HSTU_ERR_INVALID_ARG;
  }
  if (p->total_tokens > 0 && (!k_hist || !v_hist || !aligned16(k_hist) || !aligned16(v_hist)))
    return HSTU_ERR_INVALID_ARG;
  if (p->dtype != HSTU_BF16 || p->d_qk != 128 || p->d_v != 128 || p->num_heads > 16)
    return HSTU_ERR_UNSUPPORTED;
  if (static_cast<uint64_t>(p->batch) * cand_tiles(max_cands) * static_cast<uint64_t>(p->num_heads) >
      0x7FFFFFFFull)
    return HSTU_ERR_UNSUPPORTED;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0 ||
      workspace_bytes < hstu_cand_workspace_size(p, total_cands, max_cands))
    return HSTU_ERR_WORKSPACE;
  if (p->batch == 0 || total_cands == 0) return HSTU_OK;

  FwdArgs common;
  std::memset(&common, 0, sizeof(common));
  fill_common(p, static_cast<int*>(workspace), &common);
  CandArgs a;
  std::memset(&a, 0, sizeof(a));
  a.offsets = p->offsets;
  a.cand_offsets = cand_offsets;
  a.timestamps = p->timestamps;
  a.cand_ts = cand_timestamps;
  a.rab_pos = p->rab_pos;
  a.rab_time = p->rab_time;
  a.q = q; a.k = k; a.v = v; a.u = u; a.y = y;
  a.ln_weight = p->ln_weight;
  a.ln_bias = p->ln_bias;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t cnt_bytes = align_up(static_cast<size_t>(p->batch) * cand_tiles(max_cands) * 4);
  a.cnt = reinterpret_cast<unsigned*>(ws + kStatusBytes);
  a.o_ws = reinterpret_cast<float*>(ws + kStatusBytes + cnt_bytes);
  a.plan_j = static_cast<int>(cand_plan_j(p));
  const size_t plan_off =
      kStatusBytes + cnt_bytes + align_up(static_cast<size_t>(total_cands) * p->num_heads * p->d_v * 4);
  if (a.plan_j > 0) a.plan = reinterpret_cast<uint32_t*>(ws + plan_off);
  if (p->batch <= kCandOrderMax)
    a.order = reinterpret_cast<int*>(
        ws + plan_off + align_up(static_cast<size_t>(a.plan_j) * total_cands * 4));
  a.status = static_cast<int*>(workspace);
  a.B = p->batch;
  a.T = p->total_tokens;
  a.C = total_cands;
  a.H = p->num_heads;
  a.max_tiles = static_cast<int>(cand_tiles(max_cands));
  a.max_seq_len = p->max_seq_len;
  a.L = common.L;
  a.nb = common.nb;
  a.norm_len = p->norm_len;
  a.eps = p->ln_eps;
  a.bt = common.bt;
  CUtensorMap tq, tk, tv;
  // With no history at all the key and value maps are never read; they are
  // encoded over the candidates so that they stay valid.
  const bool hist = p->total_tokens > 0;
  if (!make_map_3d(&tq, q, total_cands, p->num_heads, 128) ||
      !make_map_3d(&tk, hist ? k_hist : k, hist ? p->total_tokens : total_cands, p->num_heads, 128) ||
      !make_map_3d(&tv, hist ? v_hist : v, hist ? p->total_tokens : total_cands, p->num_heads, 128))
    return HSTU_ERR_CUDA;
  cudaError_t err = cudaSuccess;
  if (a.plan && hist && total_cands > 0)   // the time-plan shapes, once for all heads
    err = launch_cand_plans(a, static_cast<cudaStream_t>(stream));
  if (err == cudaSuccess) err = launch_cand_order(a, static_cast<cudaStream_t>(stream));
  if (err == cudaSuccess) err = launch_cand_sm100(a, tq, tk, tv, static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

}  // extern "C"
