// Programmatic dependent launch for the forward kernels.
//
// Every forward kernel begins with pdl_enter(): griddepcontrol.wait blocks
// until the kernel it depends on (the previous one in the stream or graph) has
// completed and its memory is visible, and only then touches memory; after
// that, griddepcontrol.launch_dependents lets the next kernel be scheduled
// while this one runs.  Ordering is therefore exactly stream ordering; what
// overlaps is the next kernel's launch and CTA scheduling.  Without the launch
// attribute both instructions are no-ops.
#pragma once

#include <atomic>

#include "tl_internal.cuh"

namespace tl {

// One-time host set-up per device: kernel attributes such as the dynamic
// shared-memory limit belong to the device's context, so a process that
// drives several GPUs sets them on each.  Bit d of `done` records device d
// (devices past 63 repeat the set-up on every call).  Concurrent first calls
// may both run `f`; it only sets attributes, so that is harmless.
template <typename Fn>
inline tl_status once_per_device(std::atomic<uint64_t>& done, Fn f) {
  int dev = 0;
  TL_CUDA(cudaGetDevice(&dev));
  const uint64_t bit = dev >= 0 && dev < 64 ? (uint64_t)1 << dev : 0;
  if (bit != 0 && (done.load(std::memory_order_acquire) & bit) != 0) return ok();
  TL_TRY(f());
  done.fetch_or(bit, std::memory_order_release);
  return ok();
}

__device__ __forceinline__ void pdl_enter() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args... args) {
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
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// The same with thread-block clusters of cluster_x CTAs along x.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block,
                                      size_t smem, cudaStream_t s, unsigned cluster_x,
                                      Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster_x;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

#define TL_LAUNCH_PDL(kernel, grid, block, smem, stream, ...)                                \
  do {                                                                                      \
    cudaError_t e_ = ::tl::launch_pdl(kernel, dim3(grid), dim3(block), (size_t)(smem),      \
                                      stream, __VA_ARGS__);                                 \
    if (e_ != cudaSuccess)                                                                  \
      return ::tl::set_error(TL_ERR_CUDA, "launch of %s failed: %s", #kernel,              \
                             cudaGetErrorString(e_));                                       \
  } while (0)

}  // namespace tl
