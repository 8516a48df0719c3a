// launch.cuh -- programmatic dependent launch (PDL) for the library's kernel sequences.
//
// A kernel launched through launch_pdl may be scheduled while the previous kernel on the stream is
// still finishing (that kernel lets it in early with pdl_trigger).  Before it touches memory that
// earlier work writes or reads, every such kernel executes pdl_wait (griddepcontrol.wait), which
// returns once the previous grid has completed and its memory operations are visible; the work
// before that point -- setup, tensor-map prefetch, L2 prefetch of weights -- overlaps the previous
// kernel's tail.  A kernel launched without the attribute passes pdl_wait at once.
#pragma once

#include <cuda_runtime.h>

#include <utility>

namespace domino {

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace domino
