// hnd_slab_go.cuh -- host dispatch of the 3D slab stage (k_mid2v2 and its
// 2-CTA form) for one conjugation sign; included by the two instantiation
// units hnd_unit_slab_fwd.cu and hnd_unit_slab_adj.cu.
#pragma once
#include "hnd_multi2.cuh"
#include "hnd_launch.h"
#include "hnd_host_util.h"

namespace hnd {

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

template <int N0, bool CONJ>
static cudaError_t mid2_n1(const ConvArgs& a, float2* zt, long long ord0, int np) {
  switch (a.n[1]) {
    case 8: return mid2_go_c<N0, 8, CONJ>(a, zt, ord0, np);
    case 16: return mid2_go_c<N0, 16, CONJ>(a, zt, ord0, np);
    case 32: return mid2_go_c<N0, 32, CONJ>(a, zt, ord0, np);
    case 64: return mid2_go_c<N0, 64, CONJ>(a, zt, ord0, np);
    case 128: return mid2_go_c<N0, 128, CONJ>(a, zt, ord0, np);
    default: return cudaErrorInvalidValue;
  }
}

template <bool CONJ>
cudaError_t launch_mid2_conj(const ConvArgs& a, float2* zt, long long ord0, int np) {
  switch (a.n[0]) {
    case 8: return mid2_n1<8, CONJ>(a, zt, ord0, np);
    case 16: return mid2_n1<16, CONJ>(a, zt, ord0, np);
    case 32: return mid2_n1<32, CONJ>(a, zt, ord0, np);
    case 64: return mid2_n1<64, CONJ>(a, zt, ord0, np);
    case 128: return mid2_n1<128, CONJ>(a, zt, ord0, np);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace hnd
