// noalloc.cu -- backward entry point that needs no caller-provided workspace.
//
// hstu_attn_bwd needs scratch device memory (its workspace).  Some callers
// cannot hand that over: processes whose device memory is already reserved
// by another allocator (a serving runtime's memory pool that owns the free
// HBM, where a fresh cudaMalloc fails or forces a device synchronisation),
// or plug-ins hosted by a framework that forbids direct CUDA allocation.
// For them this file keeps the scratch in a fixed-size array in device
// global memory, reserved when the library is loaded on a device and held
// until the process exits, and forwards to the regular backward.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "hstu.h"
#include "internal.h"

namespace {

// Size of the built-in scratch: problems whose backward workspace
// (hstu_attn_workspace_size(p, 1)) exceeds it are rejected.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // 16 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code
// the array's name only stands in for it, so the address is looked up once
// per device, with that device current, and cached.
hstu_status_t scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HSTU_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return HSTU_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return HSTU_OK;
}

}  // namespace

extern "C" HSTU_API hstu_status_t hstu_attn_bwd_noalloc(
    const hstu_problem_t* p, const void* dy, const void* q, const void* k, const void* v,
    const void* u, const float* o_save, const float* ln_mean, const float* ln_rstd, void* dq,
    void* dk, void* dv, void* du, float* d_rab_pos, float* d_rab_time, float* d_ln_weight,
    float* d_ln_bias, void* stream) {
  // The same argument checks as hstu_attn_bwd first, so that a rejected call
  // returns the same status and leaves nothing queued on the stream.
  hstu_status_t st = hstu::check_bwd_args(p, dy, q, k, v, u, o_save, ln_mean, ln_rstd, dq, dk,
                                          dv, du, d_rab_pos, d_rab_time, d_ln_weight, d_ln_bias);
  if (st != HSTU_OK) return st;
  const size_t need = hstu_attn_workspace_size(p, 1);
  if (need == 0) return HSTU_ERR_INVALID_ARG;            // the problem itself is invalid
  if (need > kNoAllocScratchBytes) return HSTU_ERR_WORKSPACE;
  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != HSTU_OK) return st;
  // The array keeps the previous call's contents; the device status word at
  // its start must begin at zero.  Everything else the backward clears itself.
  if (cudaMemsetAsync(scratch, 0, sizeof(int), static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return HSTU_ERR_CUDA;
  return hstu_attn_bwd(p, dy, q, k, v, u, o_save, ln_mean, ln_rstd, dq, dk, dv, du, d_rab_pos,
                       d_rab_time, d_ln_weight, d_ln_bias, scratch, kNoAllocScratchBytes, stream);
}
