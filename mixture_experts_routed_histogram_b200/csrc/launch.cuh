// launch.cuh -- kernel launches with programmatic dependent launch (PDL): a kernel may
// start on free SMs while its predecessor on the stream is finishing, runs its prologue
// (barrier init, TMEM allocation, tensor-map prefetch), and waits in pdl_wait() until the
// predecessor has completed and its memory is visible before it touches any global data
// the predecessor produces or reads.  Every kernel signals pdl_launch_dependents() right
// after its own pdl_wait(): the successor's CTAs are then scheduled as soon as SM resources
// free up (the persistent GEMMs' tail wave), which is safe because the successor's
// pdl_wait() still waits for this grid's completion.
#pragma once

#include <cuda_runtime.h>

#include <utility>

namespace moe {

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                     cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace moe
