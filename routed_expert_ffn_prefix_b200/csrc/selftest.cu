// selftest.cu -- exercises the bounded device wait on a barrier that nothing
// completes, so failure detection can be tested without hanging a GPU: the
// wait gives up after timeout_ns, records MOE_ERR_DEVICE_TIMEOUT and the
// kernel returns normally.
#include "kernels.h"

namespace moe {

namespace {

__global__ void selftest_timeout_kernel(DevStatus* st, uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtx wc{st, &abort_flag, timeout_ns, SITE_SELFTEST};
    mbar_wait(&bar, 0, wc, 0);  // no thread ever arrives: returns false after timeout_ns
  }
  __syncthreads();
}

}  // namespace

cudaError_t launch_selftest_timeout(DevStatus* st, uint64_t timeout_ns, cudaStream_t s) {
  selftest_timeout_kernel<<<1, 32, 0, s>>>(st, timeout_ns);
  return cudaGetLastError();
}

}  // namespace moe
