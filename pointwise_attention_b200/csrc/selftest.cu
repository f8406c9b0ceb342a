// selftest.cu -- device self-test of the bounded-wait error path.
//
// One thread initialises an mbarrier that nothing ever arrives on and waits on
// it with the same bounded wait the attention kernels use.  The wait gives up
// after the given budget, the kernel records the timeout bit in the status
// word and returns, and the context stays usable.  No fault, trap or hang is
// involved: this is how the timeout reporting is tested on a shared GPU.
#include "hstu.h"
#include "internal.h"
#include "ptx.cuh"

namespace hstu {
namespace {

__global__ void wait_never_kernel(int* status, unsigned long long budget_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!mbar_wait(b, 0, nullptr, budget_ns)) atomicOr(status, kStatusTimeout);
    // Complete the phase so the barrier is left in a consistent state.
    mbar_arrive(b);
  }
}

}  // namespace
}  // namespace hstu

extern "C" HSTU_API hstu_status_t hstu_selftest_wait_timeout(void* workspace, uint64_t budget_ns,
                                                             void* stream) {
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % 256) != 0) return HSTU_ERR_WORKSPACE;
  if (budget_ns == 0 || budget_ns > 5000000000ull) return HSTU_ERR_INVALID_ARG;
  hstu::wait_never_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<int*>(workspace), static_cast<unsigned long long>(budget_ns));
  return cudaGetLastError() == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}
