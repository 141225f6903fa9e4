// launch.cuh -- programmatic dependent launch: a kernel launched this way may
// be scheduled while its predecessor on the stream is still running; it runs
// griddepcontrol.wait before reading the predecessor's results.
#pragma once

#include <cuda_runtime.h>

namespace moe {

// Programmatic dependent launch: wait until the preceding kernel on the stream
// has completed and its memory is visible (a no-op for a normal launch).
__device__ __forceinline__ void wait_prior_grid() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Let the next kernel on the stream (launched programmatically) be scheduled
// now rather than when this CTA exits.  Called after this CTA's own
// wait_prior_grid, so a kernel that starts early can rely on every kernel
// before this one having finished and flushed its results.
__device__ __forceinline__ void trigger_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Launch with programmatic stream serialisation: the kernel may be scheduled
// before its predecessor on the stream has finished; it waits with
// griddepcontrol.wait before reading the predecessor's results.
template <typename... Args>
inline void launch_dependent(void (*fn)(Args...), int grid, int block, size_t smem, cudaStream_t s,
                             const Args &...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3((unsigned)block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, fn, args...);
}

}  // namespace moe
