// Self-test of the bounded device wait that every kernel of the library uses:
// one CTA whose two waiting threads (in different warps) wait on an mbarrier
// that nothing completes.  The first wait gives up after its bound
// (kWaitLimitNs), sets the CTA's abort flag and records a timeout in the plan's
// status word; the other waiter sees the flag and gives up too; the kernel
// returns.  Nothing is left waiting and the context stays usable.
#include "sm100.cuh"
#include "vsa_internal.h"

namespace vsa {
namespace {
using namespace sm100;

__global__ void __launch_bounds__(64, 1) bounded_wait_kernel(unsigned int* status, int* result) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if ((threadIdx.x & 31) == 0) {
    // no thread ever arrives on the barrier: phase 0 never completes
    const bool ok = wait_bar(b, 0, &abort_flag, status, 90 + threadIdx.x / 32);
    result[threadIdx.x / 32] = ok ? 1 : 0;
  }
}

}  // namespace

cudaError_t launch_bounded_wait_check(unsigned int* status, int* result, cudaStream_t stream) {
  bounded_wait_kernel<<<1, 64, 0, stream>>>(status, result);
  return cudaGetLastError();
}

}  // namespace vsa
