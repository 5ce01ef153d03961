// HSTU block stack (placeholder until the GEMM kernels land).
#include "block.h"

namespace hstu {
size_t block_workspace_bytes(int64_t, int, int, int) { return 0; }
cudaError_t block_fwd_launch(const BlockProblem&, void*, size_t, int*, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace hstu
