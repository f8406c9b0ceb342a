// simt.cu -- CUDA-core (FMA) forward and backward of HSTU causal pointwise
// aggregated attention with fp32 arithmetic, templated on the storage type E.
//
// fp32 inputs use this path for the forward and the backward (any d_qk,
// d_v <= 128 and H*d_v <= 1024).  TF32 tensor cores (10-bit mantissa) cannot
// meet a 1e-5 relative tolerance, so fp32 is computed with plain FP32 FMAs.
// bf16 inputs use the LayerNorm/gate backward of this file (bwd_pre_rows_bf16).
//
// Same operation as the bf16 tcgen05 path ("HSTU (Generative Recommender)"
// model card, Exported PyTorch, HSTUBlock.forward; relative biases from
// "HSTU Hierarchical Sequential Transduction Units", §1 and §3; LayerNorm then
// U gate from the HSTU reproduction note's flowchart).
#include <cuda_bf16.h>

#include <algorithm>

#include "bounds.cuh"
#include "internal.h"

namespace hstu {
namespace {

constexpr int kT = 128;   // threads per block
constexpr int kMaxD = 1024;

__device__ __forceinline__ float ld(const float* p, size_t i) { return p[i]; }
__device__ __forceinline__ float ld(const __nv_bfloat16* p, size_t i) {
  return __bfloat162float(p[i]);
}
__device__ __forceinline__ void st(float* p, size_t i, float x) { p[i] = x; }
__device__ __forceinline__ void st(__nv_bfloat16* p, size_t i, float x) {
  p[i] = __float2bfloat16_rn(x);
}

__device__ __forceinline__ float silu_f(float x) { return x / (1.0f + expf(-x)); }

__device__ __forceinline__ float silu_grad_f(float x) {
  const float sg = 1.0f / (1.0f + expf(-x));
  return sg * (1.0f + x * (1.0f - sg));
}

__device__ int bucket_of(long long dt, const BucketTable& bt, int nb) {
  unsigned long long a = dt < 0 ? 0ull - static_cast<unsigned long long>(dt)
                                : static_cast<unsigned long long>(dt);
  if (a < 1ull) a = 1ull;
  const long long aa =
      static_cast<long long>(a > 0x7FFFFFFFFFFFFFFFull ? 0x7FFFFFFFFFFFFFFFull : a);
  int k = 0;
  while (k + 1 < nb && aa >= bt.thr[k + 1]) ++k;   // linear scan: this path is not the hot one
  return k;
}

__device__ __forceinline__ float block_sum(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
  for (int i = 0; i < kT / 32; ++i) t += red[i];
  return t;
}

// Locates the sequence of token t: offsets[b] <= t < offsets[b+1].
__device__ __forceinline__ int seq_of(const int32_t* off, int B, int t) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ bool seq_ok(const int32_t* off, int b, int T, int max_len, int L,
                                       bool has_pos, int* s, int* n) {
  *s = off[b];
  *n = off[b + 1] - *s;
  return !(*s < 0 || *n < 0 || *s + *n > T || *n > max_len || (has_pos && *n > L));
}

__device__ __forceinline__ float bias_at(const float* rab_pos, int L, const float* rab_time, int nb,
                                         const int64_t* ts, const BucketTable& bt, int h, int s,
                                         int i, int j) {
  float bias = 0.f;
  if (rab_pos) bias += rab_pos[static_cast<size_t>(h) * (2 * L - 1) + (i - j) + L - 1];
  if (rab_time) bias += rab_time[h * nb + bucket_of(ts[s + i] - ts[s + j], bt, nb)];
  return bias;
}

// One block per output token row: all heads, then the LayerNorm and gate.
template <typename E>
__global__ void __launch_bounds__(kT) fwd_simt(const FwdArgs a) {
  __shared__ float o_row[kMaxD];
  __shared__ float q_s[128];
  __shared__ float a_s[kT];
  __shared__ float red[kT / 32];
  const int t = blockIdx.x;
  const int b = seq_of(a.offsets, a.B, t);
  int s, n;
  if (!seq_ok(a.offsets, b, a.T, a.max_seq_len, a.L, a.rab_pos != nullptr, &s, &n) || t - s >= n) {
    if (threadIdx.x == 0) atomicOr(a.status, kStatusBadOffsets);
    return;
  }
  const int i = t - s, H = a.H, dqk = a.d_qk, dv = a.d_v, D = H * dv;
  const float nrm = a.norm_len > 0 ? static_cast<float>(a.norm_len) : static_cast<float>(n);
  const E* q = static_cast<const E*>(a.q);
  const E* k = static_cast<const E*>(a.k);
  const E* v = static_cast<const E*>(a.v);
  for (int h = 0; h < H; ++h) {
    __syncthreads();
    for (int c = threadIdx.x; c < dqk; c += kT) q_s[c] = ld(q, (static_cast<size_t>(t) * H + h) * dqk + c);
    float acc = 0.f;   // thread c < dv accumulates O[h][c]
    for (int j0 = 0; j0 <= i; j0 += kT) {
      __syncthreads();
      const int j = j0 + threadIdx.x;
      float av = 0.f;
      if (j <= i) {
        const size_t kj = (static_cast<size_t>(s + j) * H + h) * dqk;
        float dot = 0.f;
        for (int c = 0; c < dqk; ++c) dot = fmaf(q_s[c], ld(k, kj + c), dot);
        dot += bias_at(a.rab_pos, a.L, a.rab_time, a.nb, a.timestamps, a.bt, h, s, i, j);
        av = silu_f(dot) / nrm;
      }
      a_s[threadIdx.x] = av;
      __syncthreads();
      const int jn = min(kT, i + 1 - j0);
      if (threadIdx.x < dv)
        for (int jj = 0; jj < jn; ++jj)
          acc = fmaf(a_s[jj], ld(v, (static_cast<size_t>(s + j0 + jj) * H + h) * dv + threadIdx.x),
                     acc);
    }
    if (threadIdx.x < dv) o_row[h * dv + threadIdx.x] = acc;
  }
  __syncthreads();
  float part = 0.f;
  for (int c = threadIdx.x; c < D; c += kT) part += o_row[c];
  const float mean = block_sum(part, red) / static_cast<float>(D);
  part = 0.f;
  for (int c = threadIdx.x; c < D; c += kT) {
    const float d0 = o_row[c] - mean;
    part = fmaf(d0, d0, part);
  }
  const float var = block_sum(part, red) / static_cast<float>(D);
  const float rstd = 1.0f / sqrtf(var + a.eps);
  const E* u = static_cast<const E*>(a.u);
  E* y = static_cast<E*>(a.y);
  for (int c = threadIdx.x; c < D; c += kT) {
    const size_t o = static_cast<size_t>(t) * D + c;
    const float w = a.ln_weight ? a.ln_weight[c] : 1.f, bb = a.ln_bias ? a.ln_bias[c] : 0.f;
    st(y, o, fmaf((o_row[c] - mean) * rstd, w, bb) * silu_f(ld(u, o)));
    if (a.o_save) a.o_save[o] = o_row[c];
  }
  if (threadIdx.x == 0 && a.ln_mean) {
    a.ln_mean[t] = mean;
    a.ln_rstd[t] = rstd;
  }
}

// LayerNorm + gate backward, one block per row: dU (output) and dO (workspace,
// storage type E), with the LayerNorm weight gamma and bias beta (ones and
// zeros without tables):
//   dU = dY (gamma xhat + beta) SiLU'(U),  dxhat = dY SiLU(U) gamma,
//   dO = rstd (dxhat - mean(dxhat) - xhat mean(dxhat xhat)),
//   d_gamma += dY SiLU(U) xhat,  d_beta += dY SiLU(U)  (fp32 atomics).
template <typename E>
__global__ void __launch_bounds__(kT) bwd_pre_simt(const BwdArgs a) {
  __shared__ float red[kT / 32];
  const int t = blockIdx.x;
  const int D = a.H * a.d_v;
  const float mean = a.ln_mean[t], rstd = a.ln_rstd[t];
  const E* dy = static_cast<const E*>(a.dy);
  const E* u = static_cast<const E*>(a.u);
  E* du = static_cast<E*>(a.du);
  E* dO = static_cast<E*>(a.dO);
  float m1 = 0.f, m2 = 0.f;
  for (int c = threadIdx.x; c < D; c += kT) {
    const size_t o = static_cast<size_t>(t) * D + c;
    const float w = a.ln_weight ? a.ln_weight[c] : 1.f, bb = a.ln_bias ? a.ln_bias[c] : 0.f;
    const float xhat = (a.o_save[o] - mean) * rstd;
    const float uu = ld(u, o), g = ld(dy, o);
    const float dyg = g * silu_f(uu);
    const float dxh = dyg * w;
    st(du, o, g * fmaf(w, xhat, bb) * silu_grad_f(uu));
    if (a.d_ln_weight) atomicAdd(a.d_ln_weight + c, dyg * xhat);
    if (a.d_ln_bias) atomicAdd(a.d_ln_bias + c, dyg);
    m1 += dxh;
    m2 = fmaf(dxh, xhat, m2);
  }
  m1 = block_sum(m1, red) / static_cast<float>(D);
  m2 = block_sum(m2, red) / static_cast<float>(D);
  for (int c = threadIdx.x; c < D; c += kT) {
    const size_t o = static_cast<size_t>(t) * D + c;
    const float w = a.ln_weight ? a.ln_weight[c] : 1.f;
    const float xhat = (a.o_save[o] - mean) * rstd;
    const float dxh = ld(dy, o) * silu_f(ld(u, o)) * w;
    st(dO, o, rstd * (dxh - m1 - xhat * m2));
  }
}

// The same LayerNorm/gate backward for bf16 with d_v = 128, one warp per
// token row: lane l holds columns 128 c + 4 l .. +3 of every 128-column slice
// c < NC = H, so each load or store instruction of the warp covers one
// contiguous 256-byte (bf16) or 512-byte (fp32) span.  All loads of the row are
// issued before any arithmetic or store (the argument pointers may alias as far
// as the compiler knows, so it would not hoist a later slice's loads above an
// earlier slice's dU store), and the row stays in registers between the two
// reductions and the dO pass.
constexpr int kRowsPerBlock = 8;

// AFFINE: with the LayerNorm weight and bias (either may be absent: ones and
// zeros), and their gradients when asked for.  The affine form loops over
// rows (grid-stride) and keeps each lane's d_gamma / d_beta partial sums of
// its columns in registers, then adds them up per block in shared memory and
// once per block and column to the outputs (fp32 atomics).
template <int NC, bool AFFINE>
__global__ void __launch_bounds__(32 * kRowsPerBlock) bwd_pre_rows_bf16(const BwdArgs a) {
  const int lane = threadIdx.x & 31;
  constexpr int D = NC * 128;
  const __nv_bfloat16* u = static_cast<const __nv_bfloat16*>(a.u);
  const __nv_bfloat16* dy = static_cast<const __nv_bfloat16*>(a.dy);
  __nv_bfloat16* du = static_cast<__nv_bfloat16*>(a.du);
  __nv_bfloat16* dO = static_cast<__nv_bfloat16*>(a.dO);
  float gw[4 * NC], gb[4 * NC], acc_w[4 * NC], acc_b[4 * NC];
#pragma unroll
  for (int c = 0; c < NC; ++c) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int col = 128 * c + 4 * lane + e;
      gw[4 * c + e] = (AFFINE && a.ln_weight) ? __ldg(a.ln_weight + col) : 1.f;
      gb[4 * c + e] = (AFFINE && a.ln_bias) ? __ldg(a.ln_bias + col) : 0.f;
      acc_w[4 * c + e] = 0.f;
      acc_b[4 * c + e] = 0.f;
    }
  }
  const int stride = AFFINE ? static_cast<int>(gridDim.x) * kRowsPerBlock : 0;
  for (int t = blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5); t < a.T; t += stride) {
    const size_t base = static_cast<size_t>(t) * D + 4 * lane;
    float4 ov[NC];
    uint2 uv[NC], gv[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const size_t o = base + 128 * c;
      ov[c] = __ldcs(reinterpret_cast<const float4*>(a.o_save + o));
      uv[c] = __ldcs(reinterpret_cast<const uint2*>(u + o));
      gv[c] = __ldcs(reinterpret_cast<const uint2*>(dy + o));
    }
    const float mean = __ldg(a.ln_mean + t), rstd = __ldg(a.ln_rstd + t);
    float xh[4 * NC], dx[4 * NC];
    float m1 = 0.f, m2 = 0.f;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const float2 u01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&uv[c].x));
      const float2 u23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&uv[c].y));
      const float2 g01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gv[c].x));
      const float2 g23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gv[c].y));
      const float ovs[4] = {ov[c].x, ov[c].y, ov[c].z, ov[c].w};
      const float us[4] = {u01.x, u01.y, u23.x, u23.y};
      const float gs[4] = {g01.x, g01.y, g23.x, g23.y};
      float dus[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int k = 4 * c + e;
        const float x = (ovs[e] - mean) * rstd;
        const float dyg = gs[e] * silu_f(us[e]);
        const float d = AFFINE ? dyg * gw[k] : dyg;
        dus[e] = AFFINE ? gs[e] * fmaf(gw[k], x, gb[k]) * silu_grad_f(us[e])
                        : gs[e] * x * silu_grad_f(us[e]);
        if (AFFINE) {
          acc_w[k] = fmaf(dyg, x, acc_w[k]);
          acc_b[k] += dyg;
        }
        xh[k] = x;
        dx[k] = d;
        m1 += d;
        m2 = fmaf(d, x, m2);
      }
      __nv_bfloat162 d01 = __floats2bfloat162_rn(dus[0], dus[1]);
      __nv_bfloat162 d23 = __floats2bfloat162_rn(dus[2], dus[3]);
      __stcs(reinterpret_cast<uint2*>(du + base + 128 * c),
             make_uint2(*reinterpret_cast<uint32_t*>(&d01), *reinterpret_cast<uint32_t*>(&d23)));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      m1 += __shfl_xor_sync(0xffffffffu, m1, off);
      m2 += __shfl_xor_sync(0xffffffffu, m2, off);
    }
    m1 /= static_cast<float>(D);
    m2 /= static_cast<float>(D);
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      float r4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) r4[e] = rstd * (dx[4 * c + e] - m1 - xh[4 * c + e] * m2);
      __nv_bfloat162 d01 = __floats2bfloat162_rn(r4[0], r4[1]);
      __nv_bfloat162 d23 = __floats2bfloat162_rn(r4[2], r4[3]);
      *reinterpret_cast<uint2*>(dO + base + 128 * c) =
          make_uint2(*reinterpret_cast<uint32_t*>(&d01), *reinterpret_cast<uint32_t*>(&d23));
    }
    if (!AFFINE) break;
  }
  if (AFFINE && (a.d_ln_weight || a.d_ln_bias)) {
    __shared__ float s_w[D], s_b[D];
    for (int i = threadIdx.x; i < D; i += blockDim.x) {
      s_w[i] = 0.f;
      s_b[i] = 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < NC; ++c)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = 128 * c + 4 * lane + e;
        atomicAdd(&s_w[col], acc_w[4 * c + e]);
        atomicAdd(&s_b[col], acc_b[4 * c + e]);
      }
    __syncthreads();
    for (int i = threadIdx.x; i < D; i += blockDim.x) {
      if (a.d_ln_weight) atomicAdd(a.d_ln_weight + i, s_w[i]);
      if (a.d_ln_bias) atomicAdd(a.d_ln_bias + i, s_b[i]);
    }
  }
}

// dS of one (i, j) pair given q_i and dO_i in shared memory; also returns A.
template <typename E>
__device__ __forceinline__ float ds_of(const BwdArgs& a, const float* q_i, const float* dO_i,
                                      int h, int s, int i, int j, float nrm, float* a_out) {
  const E* k = static_cast<const E*>(a.k);
  const E* v = static_cast<const E*>(a.v);
  const int H = a.H, dqk = a.d_qk, dv = a.d_v;
  const size_t kj = (static_cast<size_t>(s + j) * H + h) * dqk;
  const size_t vj = (static_cast<size_t>(s + j) * H + h) * dv;
  float sc = 0.f;
  for (int c = 0; c < dqk; ++c) sc = fmaf(q_i[c], ld(k, kj + c), sc);
  sc += bias_at(a.rab_pos, a.L, a.rab_time, a.nb, a.timestamps, a.bt, h, s, i, j);
  float da = 0.f;
  for (int c = 0; c < dv; ++c) da = fmaf(dO_i[c], ld(v, vj + c), da);
  *a_out = silu_f(sc) / nrm;
  return da * silu_grad_f(sc) / nrm;
}

// dQ_i and the bias gradients: one block per (row token, head).
template <typename E>
__global__ void __launch_bounds__(kT) bwd_dq_simt(const BwdArgs a) {
  __shared__ float q_s[128], do_s[128], ds_s[kT];
  const int t = blockIdx.x, h = blockIdx.y;
  const int b = seq_of(a.offsets, a.B, t);
  int s, n;
  if (!seq_ok(a.offsets, b, a.T, a.max_seq_len, a.L, a.rab_pos != nullptr, &s, &n) || t - s >= n) {
    if (threadIdx.x == 0) atomicOr(a.status, kStatusBadOffsets);
    return;
  }
  const int i = t - s, H = a.H, dqk = a.d_qk, dv = a.d_v;
  const float nrm = a.norm_len > 0 ? static_cast<float>(a.norm_len) : static_cast<float>(n);
  const E* q = static_cast<const E*>(a.q);
  const E* k = static_cast<const E*>(a.k);
  const E* dO = static_cast<const E*>(a.dO);
  for (int c = threadIdx.x; c < dqk; c += kT) q_s[c] = ld(q, (static_cast<size_t>(t) * H + h) * dqk + c);
  for (int c = threadIdx.x; c < dv; c += kT) do_s[c] = ld(dO, static_cast<size_t>(t) * H * dv + h * dv + c);
  float acc = 0.f;
  for (int j0 = 0; j0 <= i; j0 += kT) {
    __syncthreads();
    const int j = j0 + threadIdx.x;
    float dsv = 0.f;
    if (j <= i) {
      float av;
      dsv = ds_of<E>(a, q_s, do_s, h, s, i, j, nrm, &av);
      if (a.d_rab_pos)
        atomicAdd(a.d_rab_pos + static_cast<size_t>(h) * (2 * a.L - 1) + (i - j) + a.L - 1, dsv);
      if (a.d_rab_time)
        atomicAdd(a.d_rab_time + h * a.nb +
                      bucket_of(a.timestamps[checked(a.status, s + i, a.T, BS_SIMT_TS)] -
                                    a.timestamps[checked(a.status, s + j, a.T, BS_SIMT_TS)], a.bt, a.nb),
                  dsv);
    }
    ds_s[threadIdx.x] = dsv;
    __syncthreads();
    const int jn = min(kT, i + 1 - j0);
    if (threadIdx.x < dqk)
      for (int jj = 0; jj < jn; ++jj)
        acc = fmaf(ds_s[jj], ld(k, (static_cast<size_t>(s + j0 + jj) * H + h) * dqk + threadIdx.x),
                   acc);
  }
  if (threadIdx.x < dqk)
    st(static_cast<E*>(a.dq), (static_cast<size_t>(t) * H + h) * dqk + threadIdx.x, acc);
}

// dK_j and dV_j: one block per (column token, head), over rows i >= j.
template <typename E>
__global__ void __launch_bounds__(kT) bwd_dkv_simt(const BwdArgs a) {
  __shared__ float ds_s[kT], a_s[kT];
  const int t = blockIdx.x, h = blockIdx.y;
  const int b = seq_of(a.offsets, a.B, t);
  int s, n;
  if (!seq_ok(a.offsets, b, a.T, a.max_seq_len, a.L, a.rab_pos != nullptr, &s, &n) || t - s >= n)
    return;
  const int j = t - s, H = a.H, dqk = a.d_qk, dv = a.d_v;
  const float nrm = a.norm_len > 0 ? static_cast<float>(a.norm_len) : static_cast<float>(n);
  const E* q = static_cast<const E*>(a.q);
  const E* dO = static_cast<const E*>(a.dO);
  float acc_k = 0.f, acc_v = 0.f;
  float qi[128], doi[128];
  for (int i0 = j; i0 < n; i0 += kT) {
    __syncthreads();
    const int i = i0 + threadIdx.x;
    float dsv = 0.f, av = 0.f;
    if (i < n) {
      for (int c = 0; c < dqk; ++c) qi[c] = ld(q, (static_cast<size_t>(s + i) * H + h) * dqk + c);
      for (int c = 0; c < dv; ++c) doi[c] = ld(dO, static_cast<size_t>(s + i) * H * dv + h * dv + c);
      dsv = ds_of<E>(a, qi, doi, h, s, i, j, nrm, &av);
    }
    ds_s[threadIdx.x] = dsv;
    a_s[threadIdx.x] = av;
    __syncthreads();
    const int in_ = min(kT, n - i0);
    for (int ii = 0; ii < in_; ++ii) {
      const size_t row = static_cast<size_t>(s + i0 + ii);
      if (threadIdx.x < dqk) acc_k = fmaf(ds_s[ii], ld(q, (row * H + h) * dqk + threadIdx.x), acc_k);
      if (threadIdx.x < dv) acc_v = fmaf(a_s[ii], ld(dO, row * H * dv + h * dv + threadIdx.x), acc_v);
    }
  }
  if (threadIdx.x < dqk)
    st(static_cast<E*>(a.dk), (static_cast<size_t>(t) * H + h) * dqk + threadIdx.x, acc_k);
  if (threadIdx.x < dv)
    st(static_cast<E*>(a.dv), (static_cast<size_t>(t) * H + h) * dv + threadIdx.x, acc_v);
}

template <typename E>
cudaError_t launch_bwd_simt(const BwdArgs& a, cudaStream_t stream) {
  if (a.T == 0) return cudaSuccess;
  bwd_pre_simt<E><<<a.T, kT, 0, stream>>>(a);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  bwd_dq_simt<E><<<dim3(a.T, a.H), kT, 0, stream>>>(a);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  bwd_dkv_simt<E><<<dim3(a.T, a.H), kT, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_f32_simt(const FwdArgs& a, cudaStream_t stream) {
  if (a.T == 0) return cudaSuccess;
  fwd_simt<float><<<a.T, kT, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_bwd_f32_simt(const BwdArgs& a, cudaStream_t stream) {
  return launch_bwd_simt<float>(a, stream);
}

cudaError_t launch_bwd_bf16_simt(const BwdArgs& a, cudaStream_t stream) {
  return launch_bwd_simt<__nv_bfloat16>(a, stream);
}

cudaError_t launch_bwd_pre_bf16(const BwdArgs& a, cudaStream_t stream) {
  if (a.T == 0) return cudaSuccess;
  if (a.d_v == 128 && a.H >= 1 && a.H <= 8) {
    const bool affine = a.ln_weight || a.ln_bias || a.d_ln_weight || a.d_ln_bias;
    unsigned blocks = static_cast<unsigned>((a.T + kRowsPerBlock - 1) / kRowsPerBlock);
    if (affine) {
      // rows loop per block: a few blocks per SM keep HBM busy, and the
      // per-block gradient sums stay few
      int sms = 148, dev = 0;
      if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
      blocks = std::min(blocks, static_cast<unsigned>(4 * sms));
    }
    const dim3 g(blocks), b(32 * kRowsPerBlock);
#define HSTU_ROWS_CASE(NC)                                                   \
  case NC:                                                                   \
    if (affine) bwd_pre_rows_bf16<NC, true><<<g, b, 0, stream>>>(a);        \
    else bwd_pre_rows_bf16<NC, false><<<g, b, 0, stream>>>(a);              \
    break;
    switch (a.H) {
      HSTU_ROWS_CASE(1)
      HSTU_ROWS_CASE(2)
      HSTU_ROWS_CASE(3)
      HSTU_ROWS_CASE(4)
      HSTU_ROWS_CASE(5)
      HSTU_ROWS_CASE(6)
      HSTU_ROWS_CASE(7)
      default:
        if (affine) bwd_pre_rows_bf16<8, true><<<g, b, 0, stream>>>(a);
        else bwd_pre_rows_bf16<8, false><<<g, b, 0, stream>>>(a);
        break;
    }
#undef HSTU_ROWS_CASE
  } else {
    bwd_pre_simt<__nv_bfloat16><<<a.T, kT, 0, stream>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace hstu
