// hnd_bounds.cuh -- the index-checked build (HYENA_ND_BOUNDS).
//
// In the normal build HND_G(p) and HND_S(p) are the pointer p itself and cost
// nothing.  Built with -DHYENA_ND_BOUNDS (and relocatable device code), every
// access the kernels make to a caller buffer (HND_G) or to shared memory
// (HND_S) goes through a check first:
//   * a shared pointer must lie, with all the bytes accessed, inside the
//     CTA's dynamic shared memory;
//   * a global pointer must lie inside one of the buffers the current library
//     call registered (activations, spectrum, workspace, outputs, weights).
// A failed check records HYENA_ND_ERR_DEVICE_BOUNDS in the call's status
// word (the first one recorded wins) and redirects the access to a harmless
// dummy location, so the kernel never touches memory it does not own, never
// traps and reaches every barrier it would have reached.  The host reads the
// code with hyena_nd_device_status.  The checked build is for tests: it is
// slower, and its kernels are otherwise the same source as the product's.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace hnd {

constexpr int kBoundsMax = 16;

struct BoundsTable {
  unsigned long long base[kBoundsMax];
  unsigned long long bytes[kBoundsMax];
  int n;
  int* status;
};

#ifdef HYENA_ND_BOUNDS

// One table for the whole library (relocatable device code), written by the
// host at the start of every call (stream-ordered).
extern __device__ BoundsTable g_bounds;
extern __device__ __align__(16) unsigned char g_bounds_dummy[256];

__device__ __forceinline__ bool bounds_ok(const void* p, size_t nbytes) {
  if (__isShared(p)) {
    extern __shared__ __align__(16) unsigned char hnd_dyn_smem[];
    const uint32_t off = static_cast<uint32_t>(__cvta_generic_to_shared(p));
    const uint32_t base = static_cast<uint32_t>(__cvta_generic_to_shared(hnd_dyn_smem));
    uint32_t dyn;
    asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
    return off >= base && off + nbytes <= base + dyn;
  }
  const unsigned long long a = reinterpret_cast<unsigned long long>(p);
  for (int i = 0; i < g_bounds.n; ++i)
    if (a >= g_bounds.base[i] && a + nbytes <= g_bounds.base[i] + g_bounds.bytes[i]) return true;
  return false;
}

template <class T>
__device__ __forceinline__ T* bounds_check(T* p) {
  if (bounds_ok(p, sizeof(T))) return p;
  int* st = g_bounds.status;
  if (st) atomicCAS(st, 0, 7 /* HYENA_ND_ERR_DEVICE_BOUNDS */);
  return reinterpret_cast<T*>(g_bounds_dummy);
}

// A byte range [p, p + nbytes) that an asynchronous copy will touch: true if
// it may be issued; otherwise records the error.
__device__ __forceinline__ bool bounds_range(const void* p, size_t nbytes) {
  if (bounds_ok(p, nbytes)) return true;
  int* st = g_bounds.status;
  if (st) atomicCAS(st, 0, 7 /* HYENA_ND_ERR_DEVICE_BOUNDS */);
  return false;
}

#define HND_G(p) (::hnd::bounds_check(p))
#define HND_S(p) (::hnd::bounds_check(p))
#define HND_RANGE_OK(p, n) (::hnd::bounds_range((p), (n)))

#else

#define HND_G(p) (p)
#define HND_S(p) (p)
#define HND_RANGE_OK(p, n) (true)

#endif

// Host side: the buffers of the current call (no-ops in the normal build).
struct BoundsList {
  const void* ptr[kBoundsMax];
  size_t bytes[kBoundsMax];
  int n = 0;
  void add(const void* p, size_t b) {
    if (p && b && n < kBoundsMax) {
      ptr[n] = p;
      bytes[n] = b;
      ++n;
    }
  }
};
// Upload the list (and the status word to record in) for the kernels the
// call is about to enqueue on `st`.  Normal build: does nothing.
cudaError_t bounds_register(const BoundsList& list, int* status, cudaStream_t st);

}  // namespace hnd
