// Programmatic dependent launch (sm_90 and later): a kernel launched with the
// programmatic-stream-serialization attribute may start once every CTA of the
// kernel before it in the stream has signalled (or exited), instead of when
// that kernel has finished.  The dependent kernel must wait (griddep_wait)
// before it touches anything the earlier kernel writes; work that does not
// depend on it -- here, the TMA loads of Q and K, which the positions kernels
// never touch -- overlaps the earlier kernel's tail.
//
// Only kernels launched behind one of this library's own kernels use the
// attribute: a caller's kernel may signal early while it is still writing the
// Q/K that a dependent kernel would load before its wait.
#pragma once

#include <cuda_runtime.h>

#include <utility>

namespace cmr {
namespace pdl {

// Let the kernel launched after this one in the stream start now.  Issued
// once per CTA; it does not make this CTA's later writes visible early.
__device__ __forceinline__ void launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Wait until the kernel before this one in the stream has completed and its
// writes are visible.  Returns at once when the launch had no programmatic
// predecessor.
__device__ __forceinline__ void wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Launch `kernel` on `stream`, with the programmatic-stream-serialization
// attribute when `programmatic` is set.
template <typename... Params, typename... Args>
cudaError_t launch(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                   cudaStream_t stream, bool programmatic, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = programmatic ? attr : nullptr;
  cfg.numAttrs = programmatic ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace pdl
}  // namespace cmr
