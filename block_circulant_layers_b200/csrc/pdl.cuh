// Programmatic dependent launch (sm_90+): the device side of launches made with
// programmatic stream serialization, shared by the row kernels and the layer kernels.
#pragma once

#include <cuda_runtime.h>

namespace rdfft {

// Programmatic dependent launch. griddep_wait() blocks until the grids this one
// depends on (earlier work in its stream) have completed and their memory is visible;
// a kernel launched with programmatic stream serialization calls it before its first
// global-memory access. griddep_launch_dependents() lets the next such kernel in the
// stream be scheduled once every CTA of this grid has called it or exited; that kernel
// still waits in its own griddep_wait() until this grid has completed.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}


// Launches kern<<<grid, block, smem, s>>>(args...) with programmatic stream
// serialization: it may be scheduled while the previous kernel in the stream drains,
// so kern must call griddep_wait() before it touches global memory.
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

}  // namespace rdfft
