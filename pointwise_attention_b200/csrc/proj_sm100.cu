// proj_sm100.cu -- the projections either side of HSTU's attention on sm_100a:
// TMA-staged bf16 tiles, tcgen05 MMAs with fp32 accumulators in TMEM, fused
// epilogues.
//
//   UVQK:   [U | V | Q | K] = act(X W^T + b)      X [T, E], W [H(2dv+2dqk), E]
//   OUTPUT: Z = LayerNorm_E(X + Y W_out^T + b_out)  Y [T, H dv], W_out [E, H dv]
//
// ("HSTU (Generative Recommender)" model card, HSTUBlock: uvqk = nn.Linear
// split into u, v, q, k; norm(x + out(...)) with nn.LayerNorm; the optional
// SiLU on the projection is the reproduction note's SiLU(Norm(X) W_UVQK).)
//
// A CTA computes 128 rows x NT columns: NT = 256 for UVQK (one output tensor
// per tile: every split point is a multiple of 256) and NT = E <= 512 for
// the output projection, whose epilogue needs whole rows for the LayerNorm.
// Warp 0 issues TMA loads of 128 x 64 (A) and NT x 64 (B) bf16 boxes with
// the 128-byte swizzle, warp 1 allocates TMEM and issues one 128 x 256 x 16
// MMA per 256 columns and 16-element K step (N = 256 keeps one issuing
// thread at the tensor core's rate), warps 2.. are the epilogue: S warps
// per TMEM lane quarter, one accumulator row (TMEM lane) per thread and NT/S
// columns per warp (S = 2 for UVQK, two CTAs per SM; S = 4 for the output
// projection, whose tile fills TMEM and runs one CTA per SM).  Every wait is
// bounded.
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>

#include "bounds.cuh"
#include "internal.h"
#include "ptx.cuh"
#include "tile_math.cuh"

namespace hstu {
namespace {

constexpr int kBM = 128;                   // rows per tile
constexpr int kBK = 64;                    // K elements per stage (one 128-byte swizzle row)
constexpr int kABytes = kBM * kBK * 2;     // 16 KB

enum { EPI_UVQK = 0, EPI_OUT = 1 };

// NT columns per tile; the epilogue has S warps per TMEM lane quarter, each
// taking NT / S consecutive columns of its 32 rows.
template <int EPI, int NT>
struct Cfg {
  static constexpr int S = EPI == EPI_UVQK ? 2 : 4;
  static constexpr int kThreads = 64 + 128 * S;
  static constexpr int kMinBlocks = EPI == EPI_UVQK ? 2 : 1;
  static constexpr int kCols = NT / S;   // per epilogue thread
  static constexpr int kBBytes = NT * kBK * 2;
  static constexpr int kStage = kABytes + kBBytes;
  static constexpr int kStages = 2;   // 96 KB at NT = 256 (two CTAs per SM), 160 KB at 512
  static constexpr int kOffBar = kStages * kStage;
  static constexpr int kNumBars = 2 * kStages + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffStats = kOffMisc + 16;           // float2 [S][128] row partials
  static constexpr int kSmem = kOffStats + S * kBM * 8 + 1024;
};

__device__ __forceinline__ bool wait_or_flag(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                             int* status) {
  const bool ok = mbar_wait(bar, parity, abort_flag);
  if (!ok) {
    if (status) atomicOr(status, kStatusTimeout);
    *abort_flag = 1;
  }
  return ok;
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// 32 bf16 (64 bytes) of one row, as two 32-byte or four 16-byte stores.
__device__ __forceinline__ void store_row32(__nv_bfloat16* dst, const uint32_t (&w)[16], bool v32) {
  if (v32) {
    st_global_v8(dst, reinterpret_cast<const uint32_t(&)[8]>(w[0]));
    st_global_v8(dst + 16, reinterpret_cast<const uint32_t(&)[8]>(w[8]));
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      reinterpret_cast<uint4*>(dst)[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
  }
}

// 8 consecutive fp32 values (16-byte aligned), or `fill` when p is null.
__device__ __forceinline__ void ldg_f8(const float* p, float fill, float (&v)[8]) {
  if (p) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = fill;
  }
}

template <int EPI, int NT>
__global__ void __launch_bounds__(Cfg<EPI, NT>::kThreads, Cfg<EPI, NT>::kMinBlocks)
    proj_gemm_sm100(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                    const __grid_constant__ ProjArgs a) {
  using C = Cfg<EPI, NT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto bar = [&](int i) { return sbase + C::kOffBar + 8u * i; };
  const int B_FULL = 0, B_EMPTY = C::kStages, B_TFULL = 2 * C::kStages;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  // UVQK: x = column block, y = row tile, so CTAs resident together share one
  // A tile through L2 (W stays L2-resident); output projection: x = row tile.
  const int m0 = static_cast<int>(EPI == EPI_UVQK ? blockIdx.y : blockIdx.x) * kBM;
  const int n0 = EPI == EPI_UVQK ? static_cast<int>(blockIdx.x) * NT : 0;
  const int nk = a.K / kBK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kNumBars; ++i) mbar_init(bar(i), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sbase + C::kOffMisc, NT);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int last[C::kStages];
      for (int s = 0; s < C::kStages; ++s) last[s] = -1;
      bool ok = true;
      for (int kb = 0; kb < nk && ok; ++kb) {
        const int st = kb % C::kStages, use = kb / C::kStages;
        if (use > 0) ok = wait_or_flag(bar(B_EMPTY + st), (use - 1) & 1, abort_flag, a.status);
        if (!ok) break;
        const uint32_t dst = sbase + st * C::kStage;
        mbar_arrive_expect_tx(bar(B_FULL + st), C::kStage);
        tma_load_2d(dst, &tm_a, bar(B_FULL + st), kb * kBK, checked(a.status, m0, a.T, BS_PROJ_TMA));
#pragma unroll
        for (int nb = 0; nb < NT / 256; ++nb)
          tma_load_2d(dst + kABytes + nb * 256 * 128, &tm_b, bar(B_FULL + st), kb * kBK,
                      n0 + 256 * nb);
        last[st] = use;
      }
      if (!ok)   // let the copies already issued land before shared memory goes away
        for (int s = 0; s < C::kStages; ++s)
          if (last[s] >= 0) mbar_wait(bar(B_FULL + s), last[s] & 1, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 256, false, false);
      bool ok = true;
      for (int kb = 0; kb < nk && ok; ++kb) {
        const int st = kb % C::kStages;
        ok = wait_or_flag(bar(B_FULL + st), (kb / C::kStages) & 1, abort_flag, a.status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t sa = sbase + st * C::kStage, sb = sa + kABytes;
#pragma unroll
        for (int ks = 0; ks < kBK / 16; ++ks) {
#pragma unroll
          for (int nb = 0; nb < NT / 256; ++nb)
            mma_ss(tmem + 256u * nb, sw128_desc(sa + ks * 32, 16, 1024),
                   sw128_desc(sb + nb * 256 * 128 + ks * 32, 16, 1024), idesc,
                   (kb > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(bar(B_EMPTY + st));
      }
      mma_commit(bar(B_TFULL));   // every MMA issued has completed (or none was)
      // TMEM is released only after the MMAs issued here have finished writing it.
      mbar_wait(bar(B_TFULL), 0, nullptr);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q4 = warp & 3;                         // TMEM lane quarter of this warp
    const int cs = (warp - 2) >> 2;                  // column slice 0..S-1
    const int r = 32 * q4 + lane;                    // tile row = TMEM lane
    const int t = m0 + r;
    const bool row_ok = t < a.T;
    const int c0 = cs * C::kCols;                    // first tile column of the slice
    const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * q4) << 16) + c0;
    bool ok = wait_or_flag(bar(B_TFULL), 0, abort_flag, a.status) && !*abort_flag;
    ok = __all_sync(0xffffffffu, ok);
    if (ok) tc_fence_after();
    if (EPI == EPI_UVQK) {
      if (ok) {
        // the output tensor and column this tile starts at
        const int Nu = a.Nu, Nq = a.Nq;
        __nv_bfloat16* dst;
        int col, ld;
        if (n0 < Nu) { dst = static_cast<__nv_bfloat16*>(a.out0); col = n0; ld = Nu; }
        else if (n0 < 2 * Nu) { dst = static_cast<__nv_bfloat16*>(a.out1); col = n0 - Nu; ld = Nu; }
        else if (n0 < 2 * Nu + Nq) { dst = static_cast<__nv_bfloat16*>(a.out2); col = n0 - 2 * Nu; ld = Nq; }
        else { dst = static_cast<__nv_bfloat16*>(a.out3); col = n0 - 2 * Nu - Nq; ld = Nq; }
        __nv_bfloat16* drow = dst + static_cast<size_t>(t) * ld + col + c0;
        const float* brow = a.bias ? a.bias + n0 + c0 : nullptr;
#pragma unroll 1
        for (int c = 0; c < C::kCols / 32; ++c) {
          uint32_t v[32];
          tmem_ld32_nowait(taddr + 32u * c, v);
          tmem_wait_ld_dep(v);
          uint32_t w[16];
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            float f[8], b[8];
            ldg_f8(brow ? brow + 32 * c + 8 * g : nullptr, 0.f, b);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              f[i] = __uint_as_float(v[8 * g + i]) + b[i];
              if (a.act) {
                const float hx = 0.5f * f[i];
                f[i] = fmaf(hx, tanh_approx(hx), hx);   // SiLU(x) = x/2 (1 + tanh(x/2))
              }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) w[4 * g + i] = pack2(f[2 * i], f[2 * i + 1]);
          }
          if (row_ok) store_row32(drow + 32 * c, w, a.vec32);
        }
      }
    } else {
      // Z = LayerNorm(X + Y W^T + b): each thread reduces its slice of the row
      // (Chan's merge of 32-column chunks), the S slices of a row merge through
      // shared memory, then each thread normalises its slice.
      const __nv_bfloat16* xrow = static_cast<const __nv_bfloat16*>(a.res) +
                                  static_cast<size_t>(row_ok ? t : 0) * NT + c0;
      // R = acc + x + b for 8 columns starting at slice column j
      auto resid8 = [&](const uint32_t* v, int j, float (&f)[8]) {
        float b[8];
        ldg_f8(a.bias ? a.bias + c0 + j : nullptr, 0.f, b);
        uint4 xw = make_uint4(0u, 0u, 0u, 0u);
        if (row_ok) xw = __ldg(reinterpret_cast<const uint4*>(xrow + j));
        const uint32_t xs[4] = {xw.x, xw.y, xw.z, xw.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 x2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xs[i]));
          f[2 * i] = __uint_as_float(v[2 * i]) + x2.x + b[2 * i];
          f[2 * i + 1] = __uint_as_float(v[2 * i + 1]) + x2.y + b[2 * i + 1];
        }
      };
      float cnt = 0.f, mean = 0.f, m2 = 0.f;
      if (ok) {
#pragma unroll 1
        for (int c = 0; c < C::kCols / 32; ++c) {
          uint32_t v[32];
          tmem_ld32_nowait(taddr + 32u * c, v);
          tmem_wait_ld_dep(v);
          float f[32];
#pragma unroll
          for (int g = 0; g < 4; ++g)
            resid8(v + 8 * g, 32 * c + 8 * g, reinterpret_cast<float(&)[8]>(f[8 * g]));
          float sum = 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i) sum += f[i];
          const float mc = sum * (1.0f / 32.0f);
          float mc2 = 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float d = f[i] - mc;
            mc2 = fmaf(d, d, mc2);
          }
          const float n1 = cnt + 32.f, dl = mc - mean;
          mean += dl * (32.f / n1);
          m2 += mc2 + dl * dl * (cnt * 32.f / n1);
          cnt = n1;
        }
      }
      float2* part = reinterpret_cast<float2*>(smem + C::kOffStats);
      part[cs * kBM + r] = make_float2(mean, m2);
      named_bar_sync(1, 128 * C::S);
      float mu = 0.f, M2 = 0.f;
#pragma unroll
      for (int i = 0; i < C::S; ++i) mu += part[i * kBM + r].x;
      mu *= 1.0f / C::S;
#pragma unroll
      for (int i = 0; i < C::S; ++i) {
        const float2 pi = part[i * kBM + r];
        const float d = pi.x - mu;
        M2 += pi.y + static_cast<float>(C::kCols) * d * d;
      }
      const float rstd = 1.0f / sqrtf(M2 / static_cast<float>(NT) + a.eps);
      if (ok) {
        __nv_bfloat16* zrow = static_cast<__nv_bfloat16*>(a.out0) + static_cast<size_t>(t) * NT + c0;
#pragma unroll 1
        for (int c = 0; c < C::kCols / 32; ++c) {
          uint32_t v[32];
          tmem_ld32_nowait(taddr + 32u * c, v);
          tmem_wait_ld_dep(v);
          uint32_t w[16];
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int j = 32 * c + 8 * g;
            float f[8], gw[8], gb[8];
            resid8(v + 8 * g, j, f);
            ldg_f8(a.ln_weight ? a.ln_weight + c0 + j : nullptr, 1.f, gw);
            ldg_f8(a.ln_bias ? a.ln_bias + c0 + j : nullptr, 0.f, gb);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              w[4 * g + i] = pack2(fmaf((f[2 * i] - mu) * rstd, gw[2 * i], gb[2 * i]),
                                   fmaf((f[2 * i + 1] - mu) * rstd, gw[2 * i + 1], gb[2 * i + 1]));
          }
          if (row_ok) store_row32(zrow + 32 * c, w, a.vec32);
        }
        if (row_ok && cs == 0 && a.mean) {
          a.mean[t] = mu;
          a.rstd[t] = rstd;
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, NT);
  }
}

template <int EPI, int NT>
cudaError_t launch(const ProjArgs& a, const CUtensorMap& ta, const CUtensorMap& tb, dim3 grid,
                   cudaStream_t stream) {
  using C = Cfg<EPI, NT>;
  static std::atomic<bool> configured[64];   // per device: shared-memory opt-in done
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64 || !configured[dev].load(std::memory_order_acquire)) {
    err = cudaFuncSetAttribute(proj_gemm_sm100<EPI, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               C::kSmem);
    if (err != cudaSuccess) return err;
    if (dev >= 0 && dev < 64) configured[dev].store(true, std::memory_order_release);
  }
  proj_gemm_sm100<EPI, NT><<<grid, C::kThreads, C::kSmem, stream>>>(ta, tb, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_uvqk_sm100(const ProjArgs& a, const CUtensorMap& tx, const CUtensorMap& tw,
                              cudaStream_t stream) {
  if (a.T == 0) return cudaSuccess;
  const int N = 2 * a.Nu + 2 * a.Nq;
  const dim3 grid(static_cast<unsigned>(N / 256), static_cast<unsigned>((a.T + kBM - 1) / kBM));
  return launch<EPI_UVQK, 256>(a, tx, tw, grid, stream);
}

cudaError_t launch_out_sm100(const ProjArgs& a, const CUtensorMap& ty, const CUtensorMap& tw,
                             cudaStream_t stream) {
  if (a.T == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>((a.T + kBM - 1) / kBM));
  if (a.E == 256) return launch<EPI_OUT, 256>(a, ty, tw, grid, stream);
  if (a.E == 512) return launch<EPI_OUT, 512>(a, ty, tw, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace hstu
