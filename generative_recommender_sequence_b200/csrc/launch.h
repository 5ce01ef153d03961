// Kernel launch with programmatic dependent launch (sm_90+): the launched
// kernel's CTAs may be scheduled while the previous kernel of the stream still
// runs; each kernel launched this way calls pdl_wait() (sm100.cuh) before it
// reads anything an earlier kernel writes, and pdl_launch_dependents() to let
// the next kernel start early.
#pragma once

#include <cuda_runtime.h>

namespace hstu {

// Launches `kernel` on `stream` with programmatic dependent launch enabled, so
// its CTAs may be scheduled while the previous kernel of the stream finishes;
// the kernel calls pdl_wait() before reading that kernel's results.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// The same with 2-CTA clusters along x (grid.x even): CTAs 2k and 2k + 1 form
// one cluster.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent_pairs(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                   cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace hstu
