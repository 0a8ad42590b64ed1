// Instantiation: the 3D slab stage with the conjugate spectrum (the adjoint of
// the backward).
#include "hnd_slab_go.cuh"

namespace hnd {
cudaError_t launch_mid2_adj(const ConvArgs& a, float2* zt, long long ord0, int np) {
  return launch_mid2_conj<true>(a, zt, ord0, np);
}
}  // namespace hnd
