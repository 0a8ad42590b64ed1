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

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel on the stream finishes; it must wait for that grid
// (griddepcontrol.wait) before touching memory the previous work wrote.
// `early` = false launches normally (the kernel's griddepcontrol calls are
// then no-ops).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(bool early, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = early ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace hnd

// Switch over the power-of-two extents 8..256 (LIST_N) or 8..128 (LIST_S).
#define HND_CASE_N(n, BODY) \
  case n: {                 \
    constexpr int NV = n;   \
    BODY;                   \
  }
