// Self-test of the kernels' failure path: every wait in this library is
// bounded (kWaitLimitNs); when it runs out the waiting thread raises its
// CTA's abort flag, writes QLORA_ERR_TIMEOUT to the caller's device status and
// returns, so the kernel ends and the context stays usable. This kernel makes
// one such wait run out on purpose: one thread waits on an mbarrier that
// nothing arrives on, through the same mbar_wait the GEMMs use.
#include "qlora_device.cuh"

namespace qlora {
namespace {

__global__ void bounded_wait_selftest_kernel(int32_t *status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncwarp();
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile int *af = &abort_flag;
    (void)mbar_wait(&bar, 0, af, status);   // phase 0 never completes: gives up after the limit
  }
  __syncwarp();   // the warp is reconverged before the aligned CTA barrier
  __syncthreads();
}

}  // namespace

cudaError_t launch_bounded_wait_selftest(int32_t *status, cudaStream_t st) {
  bounded_wait_selftest_kernel<<<1, 32, 0, st>>>(status);
  return cudaGetLastError();
}

}  // namespace qlora
