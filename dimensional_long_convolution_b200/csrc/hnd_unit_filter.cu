// Filter spectrum (call 1), spectrum layout conversion, diagnostics.
#include "hnd_kernels.cuh"
#include "hnd_multi2.cuh"
#include "hnd_filter2.cuh"
#include "hnd_launch.h"
#include "hnd_host_util.h"

namespace hnd {

static SpecDims make_dims(int ndim, const int* n) {
  SpecDims d;
  d.ndim = ndim;
  for (int a = 0; a < 3; ++a) d.n[a] = a < ndim ? n[a] : 1;
  return d;
}

static unsigned grid_for(long long work, int threads) {
  long long b = (work + threads - 1) / threads;
  if (b < 1) b = 1;
  if (b > 148LL * 32) b = 148LL * 32;
  return static_cast<unsigned>(b);
}

template <int HP>
static cudaError_t filter_mlp_go(const hnd2::FilterMlpArgs& fa, long long noff, cudaStream_t st) {
  auto kern = hnd2::k_filter_mlp2<HP>;
  cudaError_t e = ensure_smem(kern, hnd2::FilterSmem<HP>::bytes(96));     // the largest feature count
  if (e != cudaSuccess) return e;
  const long long blocks = (noff + hnd2::kFO - 1) / hnd2::kFO;
  kern<<<static_cast<unsigned>(blocks), hnd2::kFT, hnd2::FilterSmem<HP>::bytes(fa.fin), st>>>(fa);
  return cudaGetLastError();
}

// Full transform of length 2N along one axis of the filter grid.
template <int N>
static cudaError_t fft_axis_go(float2* grid, long long stride, long long npen, cudaStream_t st) {
  auto kern = hnd2::k_fft_axis2<N>;
  const size_t sm = hnd2::AxisSmem<N>::kBytes;
  cudaError_t e = ensure_smem(kern, sm);
  if (e != cudaSuccess) return e;
  const long long per_cta = (hnd2::kAT / 32) * (32 / hnd2::P2<N>::G);
  long long blocks = (npen + per_cta - 1) / per_cta;
  if (blocks > 148LL * 16) blocks = 148LL * 16;
  kern<<<static_cast<unsigned>(blocks), hnd2::kAT, sm, st>>>(grid, stride, npen);
  return cudaGetLastError();
}

cudaError_t launch_filter_chunk(const FilterLaunch& f, int ndim, const int* n, int c0, int nc, float2* grid,
                                void* spectrum, cudaStream_t st) {
  const SpecDims d = make_dims(ndim, n);
  long long gsz = 1, noff = 1;
  for (int a = 0; a < ndim; ++a) {
    gsz *= 2 * n[a];
    noff *= 2 * n[a] - 1;
  }
  cudaError_t e = cudaMemsetAsync(grid, 0, sizeof(float2) * gsz * nc, st);
  if (e != cudaSuccess) return e;
  hnd2::FilterMlpArgs fa;
  fa.W1 = f.W1;
  fa.b1 = f.b1;
  fa.W2 = f.W2;
  fa.b2 = f.b2;
  fa.alpha = f.alpha;
  fa.num_freqs = f.num_freqs;
  fa.hidden = f.hidden;
  fa.fin = 2 * f.num_freqs * ndim;
  fa.decay_scale = f.decay_scale;
  fa.window = f.window;
  fa.ndim = ndim;
  for (int a = 0; a < 3; ++a) fa.n[a] = a < ndim ? n[a] : 1;
  fa.c0 = c0;
  fa.nc = nc;
  fa.grid = grid;
  const int HP = (f.hidden + 31) / 32 * 32;
  e = HP <= 32 ? filter_mlp_go<32>(fa, noff, st)
      : HP <= 64 ? filter_mlp_go<64>(fa, noff, st)
      : HP <= 96 ? filter_mlp_go<96>(fa, noff, st)
                 : filter_mlp_go<128>(fa, noff, st);
  if (e != cudaSuccess) return e;
  long long stride = gsz;
  for (int a = 0; a < ndim; ++a) {
    stride /= 2 * n[a];
    const long long npen = gsz * nc / (2 * n[a]);
    switch (n[a]) {
      case 8: e = fft_axis_go<8>(grid, stride, npen, st); break;
      case 16: e = fft_axis_go<16>(grid, stride, npen, st); break;
      case 32: e = fft_axis_go<32>(grid, stride, npen, st); break;
      case 64: e = fft_axis_go<64>(grid, stride, npen, st); break;
      case 128: e = fft_axis_go<128>(grid, stride, npen, st); break;
      case 256: e = fft_axis_go<256>(grid, stride, npen, st); break;
      default: e = cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
  }
  const long long per = spec_per_channel(d);
  const float scale = static_cast<float>(1.0 / static_cast<double>(gsz));
  if (ndim == 2) {
    float4* out = static_cast<float4*>(spectrum) + static_cast<long long>(c0) * (per / 2);
    hnd2::k_spec_import_v2<<<grid_for(per / 2 * nc, 256), 256, 0, st>>>(grid, out, n[0], n[1], nc, 2LL * n[1],
                                                                        scale);
  } else if (ndim == 3) {
    float4* out = static_cast<float4*>(spectrum) + static_cast<long long>(c0) * (per / 2);
    hnd2::k_spec3_in<<<grid_for(per / 2 * nc, 256), 256, 0, st>>>(grid, out, n[0], n[1], n[2], nc, 2LL * n[2], scale);
  } else {
    k_spec_pack<<<grid_for(per * nc, 256), 256, 0, st>>>(grid, static_cast<float2*>(spectrum), d, c0, nc, scale);
  }
  return cudaGetLastError();
}

cudaError_t launch_spec_convert(int ndim, const int* n, long long C, const void* src, void* dst, bool to_natural,
                                cudaStream_t st) {
  const SpecDims d = make_dims(ndim, n);
  const long long total = spec_per_channel(d) * C;
  if (ndim == 3) {
    if (to_natural)
      hnd2::k_spec3_out<<<grid_for(total / 2, 256), 256, 0, st>>>(static_cast<const float4*>(src),
                                                                 static_cast<float2*>(dst), n[0], n[1], n[2], C);
    else
      hnd2::k_spec3_in<<<grid_for(total / 2, 256), 256, 0, st>>>(static_cast<const float2*>(src),
                                                                static_cast<float4*>(dst), n[0], n[1], n[2], C,
                                                                n[2] + 1, 1.0f);
    return cudaGetLastError();
  }
  if (ndim == 2) {
    if (to_natural)
      hnd2::k_spec_export_v2<<<grid_for(total / 2, 256), 256, 0, st>>>(static_cast<const float4*>(src),
                                                                      static_cast<float2*>(dst), n[0], n[1], C);
    else
      hnd2::k_spec_import_v2<<<grid_for(total / 2, 256), 256, 0, st>>>(static_cast<const float2*>(src),
                                                                      static_cast<float4*>(dst), n[0], n[1], C,
                                                                      n[1] + 1, 1.0f);
    return cudaGetLastError();
  }
  if (to_natural)
    k_spec_export<<<grid_for(total, 256), 256, 0, st>>>(static_cast<const float2*>(src), static_cast<float2*>(dst), d, C);
  else
    k_spec_import<<<grid_for(total, 256), 256, 0, st>>>(static_cast<const float2*>(src), static_cast<float2*>(dst), d, C);
  return cudaGetLastError();
}

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    cached[dev] = v;
  }
  return cached[dev];
}

cudaError_t launch_bounded_wait(int* status, const int* flag, long long limit_cycles, cudaStream_t st) {
  const long long max_it = limit_cycles / 1000 + 16;
  k_bounded_wait<<<1, 32, 0, st>>>(status, flag, limit_cycles, max_it);
  return cudaGetLastError();
}

}  // namespace hnd
