// Kernel launch with programmatic dependent launch (sm_90+): the launched
// kernel's CTAs may be scheduled while the previous kernel of the stream still
// runs; each kernel launched this way calls pdl_wait() (sm100.cuh) before it
// reads anything an earlier kernel writes, and pdl_launch_dependents() to let
// the next kernel start early.
#pragma once

#include <cuda_runtime.h>

namespace hstu {

// Launches `kernel` on `stream`; with `pdl` the launch carries programmatic
// dependent launch, so its CTAs may be scheduled while the previous kernel of
// the stream finishes (the kernel calls pdl_wait() before reading that
// kernel's results).  Without it the launch is an ordinary stream-ordered one
// and the kernel's pdl_wait() / pdl_launch_dependents() return at once.
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(bool pdl, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// The programmatic-dependent form, used by every kernel of the serving chain.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t stream, Args&&... args) {
  return launch_kernel(true, kernel, grid, block, smem, stream, static_cast<Args&&>(args)...);
}

}  // namespace hstu
