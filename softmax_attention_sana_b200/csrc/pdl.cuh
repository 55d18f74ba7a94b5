// Programmatic dependent launch helpers (griddepcontrol, sm_90+) for the
// kernels that chain within one library call.
#pragma once

#include <cuda_runtime.h>

#include <utility>

namespace sana {

// A kernel launched with launch_dependent() may start while the previous
// kernel in the stream is still running; it must call griddep_wait() before it
// touches anything that earlier work writes or reads, and on every path (a grid
// that never waits would let its own successor overtake its predecessor).
// griddep_wait() returns at once in a grid launched the ordinary way.
// griddep_launch_next() lets the next kernel's CTAs be scheduled before this
// grid ends; it is a no-op when the next launch is an ordinary one.
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_next() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                    cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace sana
