// Diagnostic entry point: one bounded on-device wait that nothing completes.
//
// Every wait inside the library's kernels (on an mbarrier: a bulk copy, a
// tensor-core commit, another warp) gives up after a bounded number of polls,
// writes KDA_DEVICE_TIMEOUT into the workspace status word and lets the kernel
// return instead of hanging.  This kernel runs exactly that path on an
// mbarrier no thread ever arrives on, so a caller can exercise its handling of
// an expired wait without faulting or hanging the GPU.
#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace gdr {
namespace {

__global__ void __launch_bounds__(32, 1) wait_timeout_kernel(int32_t *status, uint32_t max_polls) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    tc::mbar_fence_init();
    // the phase never completes: no arrival, no transaction
    tc::mbar_wait(&bar, 0, status, KDA_DEVICE_TIMEOUT, max_polls);
  }
}

}  // namespace

cudaError_t launch_wait_timeout(int32_t *status, uint32_t max_polls, cudaStream_t stream) {
  TraceScope tr("wait_timeout_kernel", stream);
  wait_timeout_kernel<<<1, 32, 0, stream>>>(status, max_polls);
  return cudaGetLastError();
}

}  // namespace gdr
