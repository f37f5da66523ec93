// Kernel launches with programmatic dependent launch (PDL).
//
// Every kernel of the library is launched with programmatic stream
// serialisation: it may be scheduled while the kernel before it on the stream
// is still finishing, so that launch latency and prologues (barrier set-up,
// tensor-memory allocation, tensor-map prefetch) overlap the predecessor's
// tail.  Each kernel calls pdl_wait() before it reads or writes global memory
// that earlier work on the stream writes or reads (the wait returns once the
// predecessor grid has completed and its writes are visible; without a
// programmatic predecessor it returns at once), and pdl_trigger() once its
// successor may be scheduled.  A successor is scheduled only after every CTA
// of this grid has triggered or exited, i.e. after all of them are resident,
// so an early successor never takes resources this grid still needs; kernels
// that allocate tensor memory trigger only after their allocation.
// Measured inside a CUDA graph of the denoising step, PDL gave no gain (the
// graph's launch gaps are already small), so it is opt-in: the DL_FLAG_PDL
// kernel flag (dl_set_kernel_flags) turns it on; otherwise kernels launch
// plainly and pdl_wait() returns at once.
#pragma once

#include <cuda_runtime.h>

#include <utility>

#include "../../include/dl.h"

namespace dl {

unsigned kernel_flags();  // api.cu

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

inline bool pdl_enabled() { return (kernel_flags() & DL_FLAG_PDL) != 0; }

template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                   Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace dl

// Launches and returns the launch error from the enclosing function.
#define DL_LAUNCH(...)                                   \
  do {                                                   \
    cudaError_t dl_le_ = ::dl::launch(__VA_ARGS__);      \
    if (dl_le_ != cudaSuccess) return dl_le_;            \
  } while (0)
