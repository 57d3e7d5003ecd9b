// Self-test of the failure path shared by the tensor-core kernels: a bounded
// mbarrier wait that nothing will ever satisfy must give up, report
// FC_DEVERR_TIMEOUT through the handle's error word and return, leaving the
// CUDA context usable.  Nothing here faults, traps or spins without a limit.
#include "fc_internal.h"
#include "ptx.cuh"

namespace fc {
namespace {

__global__ void wait_timeout_kernel(unsigned long long limit_ns, int32_t* err) {
  __shared__ unsigned long long mbar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(ptx::smem_u32(&mbar), 1);  // one arrival expected, none will come
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!ptx::mbar_wait_for(ptx::smem_u32(&mbar), 0u, &abort_flag, limit_ns))
      atomicOr(err, FC_DEVERR_TIMEOUT);
  }
}

}  // namespace

cudaError_t launch_selftest_wait_timeout(const fc_handle* h, cudaStream_t st, int limit_us) {
  wait_timeout_kernel<<<1, 32, 0, st>>>((unsigned long long)limit_us * 1000ull, h->ws.err);
  return cudaGetLastError();
}

}  // namespace fc
