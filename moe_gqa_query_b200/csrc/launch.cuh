// launch.cuh -- host helpers: raise a kernel's dynamic shared-memory limit once
// per (kernel, device, size) instead of on every launch; launch a kernel with
// programmatic dependent launch (and optionally as clusters).
#pragma once

#include <cuda_runtime.h>

#include <mutex>
#include <utility>
#include <vector>

namespace gqe {

inline cudaError_t ensure_smem(const void* kern, size_t bytes) {
  struct Entry {
    const void* kern;
    int dev;
    size_t bytes;
  };
  static std::mutex mu;
  static std::vector<Entry> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry& x : done)
      if (x.kern == kern && x.dev == dev && x.bytes >= bytes) return cudaSuccess;
  }
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  done.push_back({kern, dev, bytes});
  return cudaSuccess;
}

// Every kernel of the library is launched with programmatic stream
// serialization: it may start while the kernel before it on the stream is
// still running, does its set-up (barriers, tensor memory, descriptor
// prefetch), and waits in griddepcontrol.wait before it touches memory that
// kernel writes or reads.  cluster_x > 1 launches clusters of that many CTAs.
#ifndef GQE_PDL
#define GQE_PDL 1
#endif
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                                 int cluster_x, Args&&... args) {
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (GQE_PDL) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = (unsigned)cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace gqe
