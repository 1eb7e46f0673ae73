// Host-side helpers shared by the launchers.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include <map>
#include <mutex>
#include <utility>

namespace lsa {

// Raises `fn`'s dynamic shared-memory limit to at least `bytes` on the current
// device.  The limit is a per-device property of the kernel, so what has been
// set is remembered per (device, kernel), under a lock shared by all host
// threads; a second device gets its own cudaFuncSetAttribute call.
inline cudaError_t ensure_dyn_smem(const void* fn, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static std::mutex mu;
  static std::map<std::pair<int, const void*>, size_t> done;
  std::lock_guard<std::mutex> lock(mu);
  size_t& have = done[std::make_pair(dev, fn)];
  if (have >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e == cudaSuccess) have = bytes;
  return e;
}

template <class K>
inline cudaError_t ensure_dyn_smem(K* kernel, size_t bytes) {
  return ensure_dyn_smem(reinterpret_cast<const void*>(kernel), bytes);
}

}  // namespace lsa
