// launch.cuh -- host helper: raise a kernel's dynamic shared-memory limit once
// per (kernel, device, size) instead of on every launch.
#pragma once

#include <cuda_runtime.h>

#include <mutex>
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

}  // namespace gqe
