// launch.cuh -- kernel launches with programmatic dependent launch.
//
// Every kernel of the library is launched with the programmatic stream
// serialization attribute and starts with pdl_entry(): it waits
// (griddepcontrol.wait) until the kernel before it on the stream has
// completed and its memory is visible, before it touches global memory, and
// then lets the kernel after it launch (griddepcontrol.launch_dependents).
// Results and their stream order are those of plain launches; what overlaps
// is the next kernel's launch and scheduling with the end of this one.
// NVFP4_PDL=0 in the environment (read once per process) turns the
// attribute off.
#pragma once
#include <cuda_runtime.h>
#include <cstdlib>
#include <utility>

namespace nvfp4 {

__device__ __forceinline__ void pdl_entry() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

inline bool pdl_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("NVFP4_PDL");
    return !(v && v[0] == '0');
  }();
  return on;
}

// kernel<<<grid, block, smem, st>>>(args...) with the attribute (and, when
// cluster_x > 1, a cluster of cluster_x CTAs along x).
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                     unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace nvfp4
