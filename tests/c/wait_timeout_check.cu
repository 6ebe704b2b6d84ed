// Test-only kernel for the bounded waits of common.cuh: one CTA waits on an mbarrier that no
// thread arrives on and no copy completes, with a short limit, then waits again through the
// abort-path drain. Both waits must give up, the kernel must record GPTQ_ERR_TIMEOUT in the
// status word the way the library's kernels do, and return. Built by tests/test_gpu_failure.py.
#include "common.cuh"

namespace {

__global__ void wait_nobody_kernel(int32_t* status, unsigned long long limit_ns, int* result) {
  __shared__ uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    gptq::mbar_init(&bar, 1);
    gptq::fence_barrier_init();
  }
  __syncthreads();
  const bool landed = gptq::mbar_wait(&bar, 0, &abort_flag, limit_ns);
  if (!__syncthreads_and(landed)) {
    if (threadIdx.x == 0) {
      gptq::set_status(status, GPTQ_ERR_TIMEOUT, 99);
      const bool drained = gptq::mbar_drain(&bar, 0, limit_ns);
      result[0] = 1;                   // the wait gave up
      result[1] = drained ? 1 : 0;     // the drain must give up too (nothing will arrive)
      result[2] = abort_flag;
    }
    return;
  }
  if (threadIdx.x == 0) result[0] = 2;  // not expected: nothing arrives on the barrier
}

}  // namespace

extern "C" int wait_nobody(int32_t* status, unsigned long long limit_ns, int* result,
                           cudaStream_t stream) {
  wait_nobody_kernel<<<1, 64, 0, stream>>>(status, limit_ns, result);
  return cudaGetLastError() == cudaSuccess ? 0 : 1;
}
