// Programmatic dependent launch (sm_90 and later): a kernel launched with the
// programmatic-serialization attribute may start before the kernel ahead of it on
// the stream has finished, once every CTA of that kernel has signalled
// launch_dependents (or exited). It must wait (griddepcontrol.wait) before it reads
// anything the earlier kernel writes: the wait returns once every kernel it depends
// on has completed and its writes are visible, and at once for a kernel that was
// launched the ordinary way.
#pragma once

#include <cuda_runtime.h>

#include <utility>

namespace msa {

__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// kern<<<grid, block, smem, s>>>(args...), as a programmatic dependent of the previous
// kernel on `s` when `pdl` is set.
template <class... P, class... A>
cudaError_t launch_maybe_pdl(void (*kern)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                             A&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<A>(args)...);
}

}  // namespace msa
