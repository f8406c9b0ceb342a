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
// thread at the tensor core's rate), warps 2..5 are the epilogue, one
// accumulator row (TMEM lane) per thread.  Every wait is bounded.
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>

#include "internal.h"
#include "ptx.cuh"
#include "tile_math.cuh"

namespace hstu {
namespace {

constexpr int kBM = 128;                   // rows per tile
constexpr int kBK = 64;                    // K elements per stage (one 128-byte swizzle row)
constexpr int kThreads = 192;
constexpr int kABytes = kBM * kBK * 2;     // 16 KB

enum { EPI_UVQK = 0, EPI_OUT = 1 };

template <int NT>
struct Cfg {
  static constexpr int kBBytes = NT * kBK * 2;
  static constexpr int kStage = kABytes + kBBytes;
  static constexpr int kStages = 2;   // 96 KB at NT = 256 (two CTAs per SM), 160 KB at 512
  static constexpr int kOffBar = kStages * kStage;
  static constexpr int kNumBars = 2 * kStages + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmem = kOffMisc + 16 + 1024;
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

__device__ __forceinline__ void load_row32(const __nv_bfloat16* src, float (&f)[32]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(src) + i);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 p = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ws[j]));
      f[8 * i + 2 * j] = p.x;
      f[8 * i + 2 * j + 1] = p.y;
    }
  }
}

template <int EPI, int NT>
__global__ void __launch_bounds__(kThreads, 1)
    proj_gemm_sm100(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                    const __grid_constant__ ProjArgs a) {
  using C = Cfg<NT>;
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
        tma_load_2d(dst, &tm_a, bar(B_FULL + st), kb * kBK, m0);
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
    const int q4 = warp & 3;                         // TMEM lane quarter
    const int r = 32 * q4 + lane;
    const int t = m0 + r;
    const bool row_ok = t < a.T;
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q4) << 16;
    bool ok = wait_or_flag(bar(B_TFULL), 0, abort_flag, a.status) && !*abort_flag;
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      if (EPI == EPI_UVQK) {
        // the output tensor and column this tile starts at
        const int Nu = a.Nu, Nq = a.Nq;
        __nv_bfloat16* dst;
        int col, ld;
        if (n0 < Nu) { dst = static_cast<__nv_bfloat16*>(a.out0); col = n0; ld = Nu; }
        else if (n0 < 2 * Nu) { dst = static_cast<__nv_bfloat16*>(a.out1); col = n0 - Nu; ld = Nu; }
        else if (n0 < 2 * Nu + Nq) { dst = static_cast<__nv_bfloat16*>(a.out2); col = n0 - 2 * Nu; ld = Nq; }
        else { dst = static_cast<__nv_bfloat16*>(a.out3); col = n0 - 2 * Nu - Nq; ld = Nq; }
        __nv_bfloat16* drow = dst + static_cast<size_t>(t) * ld + col;
#pragma unroll 1
        for (int c = 0; c < NT / 32; ++c) {
          uint32_t v[32];
          tmem_ld32_nowait(tmem + lane_addr + 32u * c, v);
          tmem_wait_ld_dep(v);
          float f[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(v[i]);
          if (a.bias) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 b4 = __ldg(reinterpret_cast<const float4*>(a.bias + n0 + 32 * c) + i);
              f[4 * i] += b4.x; f[4 * i + 1] += b4.y; f[4 * i + 2] += b4.z; f[4 * i + 3] += b4.w;
            }
          }
          if (a.act) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float hx = 0.5f * f[i];
              f[i] = fmaf(hx, tanh_approx(hx), hx);   // SiLU(x) = x/2 (1 + tanh(x/2))
            }
          }
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) w[i] = pack2(f[2 * i], f[2 * i + 1]);
          if (row_ok) store_row32(drow + 32 * c, w, a.vec32);
        }
      } else {
        // Z = LayerNorm(X + Y W^T + b): pass 1 row statistics, pass 2 normalise.
        const int E = NT;
        const __nv_bfloat16* xrow = static_cast<const __nv_bfloat16*>(a.res) +
                                    static_cast<size_t>(row_ok ? t : 0) * E;
        auto chunk = [&](int c, float (&f)[32]) {
          uint32_t v[32];
          tmem_ld32_nowait(tmem + lane_addr + 32u * c, v);
          tmem_wait_ld_dep(v);
          float xr[32];
          if (row_ok) load_row32(xrow + 32 * c, xr);
#pragma unroll
          for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(v[i]) + (row_ok ? xr[i] : 0.f);
          if (a.bias) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 b4 = __ldg(reinterpret_cast<const float4*>(a.bias + 32 * c) + i);
              f[4 * i] += b4.x; f[4 * i + 1] += b4.y; f[4 * i + 2] += b4.z; f[4 * i + 3] += b4.w;
            }
          }
        };
        float cnt = 0.f, mean = 0.f, m2 = 0.f;       // Chan's merge of 32-value chunks
#pragma unroll 1
        for (int c = 0; c < E / 32; ++c) {
          float f[32];
          chunk(c, f);
          float s = 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i) s += f[i];
          const float mc = s * (1.0f / 32.0f);
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
        const float rstd = 1.0f / sqrtf(m2 / static_cast<float>(E) + a.eps);
        __nv_bfloat16* zrow = static_cast<__nv_bfloat16*>(a.out0) + static_cast<size_t>(t) * E;
#pragma unroll 1
        for (int c = 0; c < E / 32; ++c) {
          float f[32];
          chunk(c, f);
          float g[32], bb[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            g[i] = 1.f;
            bb[i] = 0.f;
          }
          if (a.ln_weight) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 w4 = __ldg(reinterpret_cast<const float4*>(a.ln_weight + 32 * c) + i);
              g[4 * i] = w4.x; g[4 * i + 1] = w4.y; g[4 * i + 2] = w4.z; g[4 * i + 3] = w4.w;
            }
          }
          if (a.ln_bias) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 b4 = __ldg(reinterpret_cast<const float4*>(a.ln_bias + 32 * c) + i);
              bb[4 * i] = b4.x; bb[4 * i + 1] = b4.y; bb[4 * i + 2] = b4.z; bb[4 * i + 3] = b4.w;
            }
          }
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            w[i] = pack2(fmaf((f[2 * i] - mean) * rstd, g[2 * i], bb[2 * i]),
                         fmaf((f[2 * i + 1] - mean) * rstd, g[2 * i + 1], bb[2 * i + 1]));
          if (row_ok) store_row32(zrow + 32 * c, w, a.vec32);
        }
        if (row_ok && a.mean) {
          a.mean[t] = mean;
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
  using C = Cfg<NT>;
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
  proj_gemm_sm100<EPI, NT><<<grid, kThreads, C::kSmem, stream>>>(ta, tb, a);
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
