// Instantiation: the 3D slab stage with the spectrum itself (forward convolution).
#include "hnd_slab_go.cuh"

namespace hnd {
cudaError_t launch_mid2_fwd(const ConvArgs& a, float2* zt, long long ord0, int np) {
  return launch_mid2_conj<false>(a, zt, ord0, np);
}
}  // namespace hnd
