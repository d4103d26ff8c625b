// dcp_diag.cu -- diagnostic entry point for the decode kernels' bounded pipeline waits.
//
// Every mbarrier wait in the decode kernels goes through mbar_wait (dcp_device.cuh): it polls
// for at most kWaitLimitNs of global time and then returns false, and the caller sets the
// kDevTimeout bit of the workspace status word instead of spinning forever.  This file lets a
// test drive that exact path without disturbing a real pipeline: one thread waits on a freshly
// initialised mbarrier that nothing ever arrives on.  No copy or product is in flight, so giving
// up is safe; the CUDA context stays usable and the status word carries the verdict.
#include "dcp_device.cuh"
#include "dcp_internal.h"

namespace dcp {
namespace {

__global__ void wait_timeout_check_kernel(int* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    if (!mbar_wait(&bar, 0)) atomicOr(status, kDevTimeout);  // phase 0 never completes
  }
}

}  // namespace
}  // namespace dcp

extern "C" DCP_API dcp_status dcp_check_wait_timeout(void* workspace, void* stream) {
  if (workspace == nullptr) return DCP_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  dcp::wait_timeout_check_kernel<<<1, 32, 0, st>>>(static_cast<int*>(workspace));
  return cudaGetLastError() == cudaSuccess ? DCP_OK : DCP_ERR_CUDA;
}
