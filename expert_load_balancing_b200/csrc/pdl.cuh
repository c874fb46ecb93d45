// pdl.cuh -- programmatic dependent launch for chains of short kernels.
//
// A kernel launched with launch_pdl may be scheduled while the kernel before
// it in the stream is still running.  It must call pdl_wait() before its
// first global memory access: the wait returns once that earlier grid has
// completed and its writes are visible, so the chain keeps stream order and
// only the launch latency overlaps.  pdl_trigger() lets the next kernel of
// the chain be scheduled; without it that happens when this grid exits.
// Both are no-ops for a kernel launched the ordinary way.
#pragma once

#include <cuda_runtime.h>

namespace kolibri {

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Launch kern<<<grid, block, smem, s>>>(args...) with programmatic stream
// serialisation, plus an optional cluster shape (cluster.x == 0: none).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       dim3 cluster, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster.x != 0) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster.x;
    attr[n].val.clusterDim.y = cluster.y;
    attr[n].val.clusterDim.z = cluster.z;
    ++n;
  }
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = n;
  const cudaError_t err = cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace kolibri
