// Kernel launch with programmatic stream serialization: the grid may be
// scheduled while the previous grid in the stream still runs, so the kernel
// must wait for that grid (griddepcontrol.wait, sm100::grid_dep_wait) before
// it touches global memory.  The kernels launched this way also issue
// griddepcontrol.launch_dependents at their start, so that the next grid's
// CTAs take SMs as this grid's leave instead of after a full launch gap.
#pragma once

#include <cuda_runtime.h>

#include <utility>

namespace sdpa {

template <typename... KernArgs, typename... Args>
inline cudaError_t launch_serialized(void (*kern)(KernArgs...), dim3 grid, dim3 block, size_t smem,
                                     cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace sdpa
