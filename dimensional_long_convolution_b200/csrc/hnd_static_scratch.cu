// hnd_static_scratch.cu -- hyena_nd_fftconv_batched_static: the batched
// convolution for callers that cannot allocate device memory.
//
// Some callers have no way to give the library a workspace: a plugin whose
// interface passes only input and output buffers, or an application that
// reserves every byte of device memory at start-up and forbids allocations
// afterwards.  This entry point serves them.  The only scratch it needs (the
// packed row spectra of the multi-pass tiers, the split grids of the long 1D
// tier) lives in a fixed array that is part of the library's device image, so
// nothing is allocated per call.
//
// Properties a caller must know:
//  * The array holds a 256-byte control area (the device status word) and
//    then kStaticScratchBytes (16 MiB) of scratch.  Every GPU that loads the
//    library keeps it until the process exits.
//  * Problems whose single (b, c) volume needs more scratch than that (8
//    bytes per voxel in the multi-pass tiers, for example a 128 x 128 x 256
//    volume; 16 bytes per token in the long 1D tier, so n > 2^20) are
//    rejected with HYENA_ND_ERR_WORKSPACE_TOO_SMALL before anything runs.
//  * The first call on a device looks up the array's device address (once
//    per device, with that device current).  Make that first call before any
//    stream capture.
//  * All calls share the one array, and it keeps whatever the previous call
//    left there.  Each call writes every intermediate it later reads, so
//    nothing needs to start at zero; the status word starts at zero when the
//    library loads and is cleared only by hyena_nd_device_status(NULL, ...).
//    Two calls whose kernels overlap on the GPU (different streams, or
//    different host threads on one device) race on the array: serialise them.
//  * Device-side errors (a bounded wait of the fused 2D kernel that gives up)
//    are recorded in the array's status word; hyena_nd_device_status with a
//    null workspace pointer reads and clears it.
//  * Nothing here calls cudaMalloc, cudaFree or any allocating routine.
#include "hyena_nd.h"
#include "hnd_bounds.cuh"
#include "hnd_launch.h"

#include <cuda_runtime.h>

#include <climits>
#include <cstdint>
#include <mutex>

namespace hnd {
cudaError_t launch_fused2d_f32(const ConvArgs& a);
cudaError_t launch_fused2d_bf16(const ConvArgs& a);
}  // namespace hnd

namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;
constexpr size_t kStaticControlBytes = 256;      // status word + padding, ahead of the scratch

// The array itself.  Host code must not pass this name to a kernel: on the
// host it is only a stand-in for the symbol.  Its device address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticControlBytes + kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the array on the current device (looked up once).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

constexpr long long kLong1DMax = 1LL << 26;    // the longest 1D grid of the library

bool pow2_in(long long x, long long lo, long long hi) { return x >= lo && x <= hi && (x & (x - 1)) == 0; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool overlaps(const void* a, const void* b, size_t n) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + n && y < x + n;
}

}  // namespace

namespace hnd {
cudaError_t static_status_word(int** out) {
  void* base = nullptr;
  const cudaError_t e = scratch_address(&base);
  if (e != cudaSuccess) return e;
  *out = static_cast<int*>(base);
  return cudaSuccess;
}
}  // namespace hnd

extern "C" HYENA_ND_API hyena_nd_status hyena_nd_fftconv_batched_static(
    const hyena_nd_problem* p, const void* q, const void* k, const void* v, const void* spectrum,
    int64_t spectrum_batch_stride, void* y, void* cuda_stream) {
  // argument checks (the same rules as hyena_nd_fftconv_batched)
  if (!p) return HYENA_ND_ERR_INVALID_ARG;
  if (p->ndim < 1 || p->ndim > 3 || p->B < 1 || p->C < 1) return HYENA_ND_ERR_INVALID_ARG;
  if (p->io_dtype != HYENA_ND_F32 && p->io_dtype != HYENA_ND_BF16) return HYENA_ND_ERR_INVALID_ARG;
  for (int a = 0; a < p->ndim; ++a)
    if (p->n[a] < 1) return HYENA_ND_ERR_INVALID_ARG;
  if (p->circular != 0 && p->circular != 1) return HYENA_ND_ERR_INVALID_ARG;
  for (int a = 0; a < p->ndim; ++a)
    if (!pow2_in(p->n[a], 8, p->ndim == 1 ? kLong1DMax : 256)) return HYENA_ND_ERR_UNSUPPORTED;
  if (p->ndim == 3 && (p->n[0] > 128 || p->n[1] > 128)) return HYENA_ND_ERR_UNSUPPORTED;
  if (p->B > INT_MAX / p->C) return HYENA_ND_ERR_UNSUPPORTED;
  if (!q || !k || !v || !spectrum || !y) return HYENA_ND_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(spectrum) || !aligned16(y))
    return HYENA_ND_ERR_MISALIGNED;
  if (spectrum_batch_stride < 0) return HYENA_ND_ERR_INVALID_ARG;
  if (spectrum_batch_stride % 16 != 0) return HYENA_ND_ERR_MISALIGNED;

  long long L = 1;
  int n[3] = {1, 1, 1};
  for (int a = 0; a < p->ndim; ++a) {
    n[a] = static_cast<int>(p->n[a]);
    L *= p->n[a];
  }
  const bool bf16 = p->io_dtype == HYENA_ND_BF16;
  const size_t act_bytes = static_cast<size_t>(p->B * p->C * L) * (bf16 ? 2 : 4);
  if (overlaps(y, q, act_bytes) || overlaps(y, k, act_bytes) || overlaps(y, v, act_bytes))
    return HYENA_ND_ERR_INVALID_ARG;

  const bool long1d = p->ndim == 1 && n[0] > 256;
  const bool fused = (p->ndim == 1 && !long1d) || hnd::fused_2d(p->ndim, n);
  // scratch per wave item: the packed row spectra of a (b, c) volume
  // (multi-pass) or the padded split grid of a channel pair (long 1D)
  const size_t per_pair = static_cast<size_t>(long1d ? 16 : 8) * static_cast<size_t>(L);
  if (!fused && per_pair > kStaticScratchBytes) return HYENA_ND_ERR_WORKSPACE_TOO_SMALL;

  void* base = nullptr;
  if (scratch_address(&base) != cudaSuccess) return HYENA_ND_ERR_CUDA;

  hnd::ConvArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.spec = spectrum;
  a.sbs = spectrum_batch_stride / 8;
  a.y = y;
  a.B = static_cast<int>(p->B);
  a.C = static_cast<int>(p->C);
  a.bf16 = bf16 ? 1 : 0;
  a.ndim = p->ndim;
  for (int i = 0; i < 3; ++i) a.n[i] = n[i];
  a.stream = static_cast<cudaStream_t>(cuda_stream);
  a.status = static_cast<int*>(base);
  float2* zt = reinterpret_cast<float2*>(static_cast<unsigned char*>(base) + kStaticControlBytes);

  hnd::BoundsList bl;
  for (const void* ptr : {q, k, v, static_cast<const void*>(y)}) bl.add(ptr, act_bytes);
  const size_t spec_bytes = hnd::spectrum_set_bytes(p->ndim, n, p->C);
  bl.add(spectrum, spectrum_batch_stride > 0
                       ? static_cast<size_t>(p->B - 1) * static_cast<size_t>(spectrum_batch_stride) + spec_bytes
                       : spec_bytes);
  bl.add(base, kStaticControlBytes + kStaticScratchBytes);
  if (hnd::bounds_register(bl, a.status, a.stream) != cudaSuccess) return HYENA_ND_ERR_CUDA;

  cudaError_t e = cudaSuccess;
  int launches = 0;
  const long long pairs = p->B * p->C;
  if (long1d) {
    const long long grids = p->B * ((p->C + 1) / 2);
    const long long wave = hnd::balanced_wave(grids, 1, per_pair, kStaticScratchBytes, false);
    e = hnd::launch_long1d(a, zt, wave, &launches);
  } else if (p->ndim == 1) {
    e = hnd::launch_rows1d(a);
    launches = 1;
  } else if (fused) {
    e = bf16 ? hnd::launch_fused2d_bf16(a) : hnd::launch_fused2d_f32(a);
    launches = 1;
  } else {
    const long long wave = hnd::balanced_wave(pairs, p->B, per_pair, kStaticScratchBytes, true);
    const int nl = n[p->ndim - 1];
    const int rp_total = static_cast<int>(L / nl / 2);
    for (long long ord0 = 0; ord0 < pairs && e == cudaSuccess; ord0 += wave) {
      const int np = static_cast<int>(pairs - ord0 < wave ? pairs - ord0 : wave);
      e = hnd::launch_rowfwd(a, nl, zt, ord0, np, rp_total);
      if (e == cudaSuccess) e = p->ndim == 2 ? hnd::launch_mid1(a, zt, ord0, np) : hnd::launch_mid2(a, zt, ord0, np);
      if (e == cudaSuccess) e = hnd::launch_rowinv(a, nl, zt, ord0, np, rp_total);
      launches += 3;
    }
  }
  if (e != cudaSuccess) return HYENA_ND_ERR_CUDA;
  hnd::note_launches(launches);
  return HYENA_ND_OK;
}
