// Instantiations: multi-pass 2D column stage on the packed two-path FFT core;
// the 3D slab stage is instantiated in hnd_unit_slab_fwd.cu (the spectrum)
// and hnd_unit_slab_adj.cu (its conjugate), which compile in parallel.
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

cudaError_t launch_mid2(const ConvArgs& a, float2* zt, long long ord0, int np) {
  return a.sconj < 0.f ? launch_mid2_adj(a, zt, ord0, np) : launch_mid2_fwd(a, zt, ord0, np);
}

}  // namespace hnd
