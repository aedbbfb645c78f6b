// Kernel launches with programmatic dependent launch: a kernel launched this
// way may be scheduled while the previous kernel on the stream is finishing.
// Every kernel of this library calls pdl_wait() before it touches memory that
// an earlier kernel may still be writing, so stream order is kept; what
// overlaps is the launch latency and the setup before that point. A kernel
// calls pdl_trigger() once the next one may be scheduled (it then waits in its
// own pdl_wait()). Both instructions are no-ops for a normal launch.
#pragma once
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "per_device.h"

namespace pkv {

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Launches still to be failed on purpose (kv_testing_fail_launches): a fake
// of a failing launch for the host-side error-path tests.
extern std::atomic<int> g_fail_launches;

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  if (g_fail_launches.load(std::memory_order_relaxed) > 0 &&
      g_fail_launches.fetch_sub(1, std::memory_order_relaxed) > 0)
    return cudaErrorLaunchFailure;
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

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) applies to the current
// device only, so it is set once per (kernel, device). `done` is the caller's
// per-kernel array of kMaxDevices flags.
template <typename F>
cudaError_t ensure_dynamic_smem(F kern, int bytes, std::atomic<uint8_t>* done) {
  int dev = 0;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  return once_per_device(dev, done, cudaSuccess, cudaErrorInvalidDevice, [&]() {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  });
}

}  // namespace pkv
