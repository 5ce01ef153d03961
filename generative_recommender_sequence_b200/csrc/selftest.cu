// Failure-detection self test: a bounded wait that runs out on purpose.
//
// Every wait in the library's kernels spins on an mbarrier with a limit on
// %globaltimer; when the limit passes, the kernel records DEV_ERR_TIMEOUT in the
// library's device error word and winds down instead of spinning forever, so
// the context stays usable and the host reads the error.  This kernel drives
// exactly that path with a barrier that nothing ever arrives on and a short
// limit.  No fault, trap or unbounded wait is involved.
#include <cuda_runtime.h>

#include "selftest.h"
#include "sm100.cuh"

namespace hstu {

namespace {

__global__ void wait_timeout_selftest_kernel(int* err_word, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  fence_mbar_init();
  // phase 0 needs one arrival, which never comes
  const unsigned long long t0 = globaltimer_ns();
  bool completed = false;
  while (!completed && globaltimer_ns() - t0 <= limit_ns) completed = mbar_try_wait(b, 0);
  if (!completed) atomicExch(err_word, DEV_ERR_TIMEOUT);
}

}  // namespace

cudaError_t wait_timeout_selftest_launch(int* err_word, int64_t limit_ns, cudaStream_t stream) {
  if (err_word == nullptr || limit_ns <= 0) return cudaErrorInvalidValue;
  wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(err_word, (unsigned long long)limit_ns);
  return cudaGetLastError();
}

}  // namespace hstu
