// Programmatic dependent launch (sm_90 and later): a chain of dependent
// kernels on one stream overlaps each launch with the tail of the kernel
// before it.  A kernel launched with launch_pdl may start while its
// predecessor is still running, so it calls pdl_wait() before it reads
// anything that predecessor wrote; pdl_wait returns once the predecessor
// grid has completed and its writes are visible (a no-op for an ordinary
// launch).  pdl_release() lets the next kernel in the stream launch as soon
// as every block of this one has started; the next kernel still waits in
// its own pdl_wait() for this one to finish, so no kernel ever waits for a
// later one.
#pragma once

#include <cuda_runtime.h>

namespace spin4d {

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_release() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... Params, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Params>(args)...);
}

}  // namespace spin4d
