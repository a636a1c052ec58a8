// Programmatic dependent launch for the library's element-wise kernels.
//
// A kernel launched with launch_pdl may start while the previous kernel in
// the stream is still running; it calls pdl_wait() before reading anything
// that kernel writes. It calls pdl_trigger() at entry, so the next kernel
// (a GEMM, which waits the same way before reading its activations) can take
// SMs as they free up and prefetch its weights meanwhile.
#pragma once

#include <cuda_runtime.h>

namespace spense {

__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), unsigned int grid, unsigned int block, size_t smem,
                       cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace spense
