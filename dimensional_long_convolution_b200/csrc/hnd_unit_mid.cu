// Instantiations: multi-pass column stages (2D pencils, 3D slabs) on the
// packed two-path FFT core.
#include "hnd_multi2.cuh"
#include "hnd_launch.h"
#include "hnd_host_util.h"

namespace hnd {

template <int N0, bool CONJ>
static cudaError_t mid1_go_c(const ConvArgs& a, float2* zt, long long ord0, int np) {
  auto kern = hnd2::k_mid1v2<N0, CONJ>;
  const size_t sm = hnd2::M1<N0>::kBytes;
  cudaError_t e = ensure_smem(kern, sm);
  if (e != cudaSuccess) return e;
  constexpr int UPB = hnd2::M1<N0>::UPB;
  const int n1 = a.n[1];
  dim3 grid(np, (n1 + UPB - 1) / UPB);
  return launch_pdl(true, kern, grid, dim3(hnd2::kTM), sm, a.stream, zt, static_cast<const float4*>(a.spec),
                    a.sbs / 2, n1, ord0, a.B, a.C);
}

// sconj = -1: the adjoint (conjugate spectrum), a separate instantiation
template <int N0>
static cudaError_t mid1_go(const ConvArgs& a, float2* zt, long long ord0, int np) {
  return a.sconj < 0.f ? mid1_go_c<N0, true>(a, zt, ord0, np) : mid1_go_c<N0, false>(a, zt, ord0, np);
}

cudaError_t launch_mid1(const ConvArgs& a, float2* zt, long long ord0, int np) {
  switch (a.n[0]) {
    case 8: return mid1_go<8>(a, zt, ord0, np);
    case 16: return mid1_go<16>(a, zt, ord0, np);
    case 32: return mid1_go<32>(a, zt, ord0, np);
    case 64: return mid1_go<64>(a, zt, ord0, np);
    case 128: return mid1_go<128>(a, zt, ord0, np);
    case 256: return mid1_go<256>(a, zt, ord0, np);
    default: return cudaErrorInvalidValue;
  }
}

template <int N0, int N1, bool CONJ>
static cudaError_t mid2_go_c(const ConvArgs& a, float2* zt, long long ord0, int np) {
  const int n2 = a.n[2];
  if (hnd2::M2<N0, N1, false>::kBytes <= kMaxSmem) {
    auto kern = hnd2::k_mid2v2<N0, N1, CONJ>;
    const size_t sm = hnd2::M2<N0, N1, false>::kBytes;
    cudaError_t e = ensure_smem(kern, sm);
    if (e != cudaSuccess) return e;
    dim3 grid(np, n2 + 1);
    return launch_pdl(true, kern, grid, dim3(hnd2::kTM), sm, a.stream, zt, static_cast<const float4*>(a.spec),
                      a.sbs / 2, n2, ord0, a.B, a.C);
  } else {
    auto kern = hnd2::k_mid2v2_pair<N0, N1, CONJ>;
    const size_t sm = hnd2::M2<N0, N1, true>::kBytes;
    cudaError_t e = ensure_smem(kern, sm);
    if (e != cudaSuccess) return e;
    dim3 grid(2 * np, n2 + 1);
    return launch_pdl(true, kern, grid, dim3(hnd2::kTM), sm, a.stream, zt, static_cast<const float4*>(a.spec),
                      a.sbs / 2, n2, ord0, a.B, a.C);
  }
}

template <int N0, int N1>
static cudaError_t mid2_go(const ConvArgs& a, float2* zt, long long ord0, int np) {
  return a.sconj < 0.f ? mid2_go_c<N0, N1, true>(a, zt, ord0, np) : mid2_go_c<N0, N1, false>(a, zt, ord0, np);
}

template <int N0>
static cudaError_t mid2_n1(const ConvArgs& a, float2* zt, long long ord0, int np) {
  switch (a.n[1]) {
    case 8: return mid2_go<N0, 8>(a, zt, ord0, np);
    case 16: return mid2_go<N0, 16>(a, zt, ord0, np);
    case 32: return mid2_go<N0, 32>(a, zt, ord0, np);
    case 64: return mid2_go<N0, 64>(a, zt, ord0, np);
    case 128: return mid2_go<N0, 128>(a, zt, ord0, np);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_mid2(const ConvArgs& a, float2* zt, long long ord0, int np) {
  switch (a.n[0]) {
    case 8: return mid2_n1<8>(a, zt, ord0, np);
    case 16: return mid2_n1<16>(a, zt, ord0, np);
    case 32: return mid2_n1<32>(a, zt, ord0, np);
    case 64: return mid2_n1<64>(a, zt, ord0, np);
    case 128: return mid2_n1<128>(a, zt, ord0, np);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace hnd
