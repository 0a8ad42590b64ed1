// hnd_host_util.h -- small host helpers for the instantiation units.
#pragma once

#include <cuda_runtime.h>

#include <mutex>
#include <set>
#include <utility>

namespace hnd {

// Raise a kernel's dynamic shared-memory limit once per device.
template <typename K>
inline cudaError_t ensure_smem(K kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  std::lock_guard<std::mutex> lk(mu);
  const auto key = std::make_pair(reinterpret_cast<const void*>(kernel), dev);
  if (done.count(key)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e == cudaSuccess) done.insert(key);
  return e;
}

}  // namespace hnd

// Switch over the power-of-two extents 8..256 (LIST_N) or 8..128 (LIST_S).
#define HND_CASE_N(n, BODY) \
  case n: {                 \
    constexpr int NV = n;   \
    BODY;                   \
  }
