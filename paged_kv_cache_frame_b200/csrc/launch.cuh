// Kernel launches with programmatic dependent launch: a kernel launched this
// way may be scheduled while the previous kernel on the stream is finishing.
// Every kernel of this library calls pdl_wait() before it touches memory that
// an earlier kernel may still be writing, so stream order is kept; what
// overlaps is the launch latency and the setup before that point. A kernel
// calls pdl_trigger() once the next one may be scheduled (it then waits in its
// own pdl_wait()). Both instructions are no-ops for a normal launch.
#pragma once
#include <cuda_runtime.h>

namespace pkv {

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
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

}  // namespace pkv
