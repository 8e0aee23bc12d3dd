// kd_selftest.cu -- a check of the library's failure reporting that faults,
// traps and hangs nothing.  One CTA waits, through the same bounded mbarrier
// wait the tensor-core kernels use, on a barrier that no thread arrives at;
// the wait gives up after a few thousand polls, records the timeout in the
// device error word and the kernel returns normally, so the context stays
// usable and kron_delta_device_status reports KD_ERR_TIMEOUT.
#include "kd_kernels.h"
#include "kd_tc.cuh"

namespace kd {

namespace {

constexpr long kSelftestPolls = 4096;

__global__ void __launch_bounds__(32) selftest_timeout_kernel(int* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    tc::mbar_init_fence();
    abort_flag = 0;
  }
  __syncthreads();
  // nothing ever arrives: phase 0 never completes
  tc::mbar_wait<false, kSelftestPolls>(&bar, 0, err, tc::kErrTimeoutLoad, &abort_flag);
}

}  // namespace

cudaError_t launch_selftest_timeout(int* err, cudaStream_t st) {
  selftest_timeout_kernel<<<1, 32, 0, st>>>(err);
  return cudaGetLastError();
}

}  // namespace kd
