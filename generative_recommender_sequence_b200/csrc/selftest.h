// Internal interface of the failure-detection self test (not part of the C ABI).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace hstu {

// One thread waits on an mbarrier that nothing completes, for at most limit_ns
// nanoseconds of %globaltimer, then records DEV_ERR_TIMEOUT in *err_word: the
// same bounded wait and error path every kernel of the library uses.
cudaError_t wait_timeout_selftest_launch(int* err_word, int64_t limit_ns, cudaStream_t stream);

}  // namespace hstu
