// launch.cuh -- kernel launch as a programmatic dependent of the previous
// kernel on the stream (the kernel must execute griddepcontrol.wait before it
// touches global memory).
#pragma once
#include <cuda_runtime.h>

#include "swa_internal.h"

namespace swa {

template <typename Kernel, typename... Args>
int launch_dependent(Kernel kernel, unsigned grid, unsigned block, size_t smem,
                     cudaStream_t stream, const Args&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return map_cuda_error(cudaLaunchKernelEx(&cfg, kernel, args...));
}

}  // namespace swa
