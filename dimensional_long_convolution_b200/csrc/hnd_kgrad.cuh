// hnd_kgrad.cuh -- the gradient with respect to the kernel values,
//   dK[c, t] = sum_b sum_{i in [0,n)^d} q[b,c,i] dy[b,c,i] u[b,c,i - t],
// t in [-(n-1), n-1]^d, u = k v: the cross-correlation of z = q dy with u,
// summed over the batch, through zero-padded transforms on the 2n grid
// (blog "Native multi-dimensional subquadratic operators via input-dependent
// long convolutions", gradient sections: the kernel gradient by correlation).
//   k_kg_pad      z or u, zero-padded into complex grids [vol][P^d]
//   (axis transforms of hnd_filter2.cuh on every grid)
//   k_kg_corr     acc_c = conj(sum_b Z_b conj(U_b)), b in order (deterministic)
//   (axis transforms again: the inverse as conj(F(conj(.))))
//   k_kg_extract  dK[c, t] = Re(acc_c)[t mod P] / prod P
// Axes are scalars (an unused axis has extent 1).
#pragma once

#include "hnd_fused2.cuh"

namespace hnd2 {

struct KgDims {
  int n0, n1, n2;       // grid (1 for unused axes)
  int P0, P1, P2;       // padded grid (1 for unused axes)
};

template <class T>
static __global__ void k_kg_pad(const T* __restrict__ a, const T* __restrict__ b, float2* __restrict__ grid,
                                KgDims d, int B, int C, int c0, int nvol) {
  const long long gsz = static_cast<long long>(d.P0) * d.P1 * d.P2;
  const long long L = static_cast<long long>(d.n0) * d.n1 * d.n2;
  const long long total = gsz * nvol;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int vv = static_cast<int>(e / gsz);
    long long r = e % gsz;
    const int s2 = static_cast<int>(r % d.P2);
    r /= d.P2;
    const int s1 = static_cast<int>(r % d.P1);
    const int s0 = static_cast<int>(r / d.P1);
    float val = 0.f;
    if (s0 < d.n0 && s1 < d.n1 && s2 < d.n2) {
      const int cl = vv / B, bb = vv % B;
      const long long idx = (static_cast<long long>(bb) * C + c0 + cl) * L + (static_cast<long long>(s0) * d.n1 + s1) * d.n2 + s2;
      val = Act<T>::ld_g(a + idx) * Act<T>::ld_g(b + idx);
    }
    grid[e] = make_float2(val, 0.f);
  }
}

// gu, gz: [ncc B][P^d] transformed grids (channel-major, sample-minor);
// acc: [ncc][P^d].
static __global__ void k_kg_corr(const float2* __restrict__ gu, const float2* __restrict__ gz,
                                 float2* __restrict__ acc, int B, int ncc, long long gsz) {
  const long long total = gsz * ncc;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long c = e / gsz, r = e % gsz;
    float re = 0.f, im = 0.f;
    for (int b = 0; b < B; ++b) {
      const long long o = (c * B + b) * gsz + r;
      const float2 z = gz[o], u = gu[o];
      re += z.x * u.x + z.y * u.y;      // z conj(u)
      im += z.y * u.x - z.x * u.y;
    }
    acc[e] = make_float2(re, -im);     // conjugated: the inverse runs as a forward transform
  }
}

static __global__ void k_kg_extract(const float2* __restrict__ acc, float* __restrict__ dK, KgDims d, int c0, int ncc,
                                    float scale) {
  const int E0 = 2 * d.n0 - 1, E1 = 2 * d.n1 - 1, E2 = 2 * d.n2 - 1;
  const long long noff = static_cast<long long>(E0) * E1 * E2;
  const long long gsz = static_cast<long long>(d.P0) * d.P1 * d.P2;
  const long long total = noff * ncc;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long c = e / noff, off = e % noff;
    long long r = off;
    const int i2 = static_cast<int>(r % E2);
    r /= E2;
    const int i1 = static_cast<int>(r % E1);
    const int i0 = static_cast<int>(r / E1);
    const int t0 = i0 - (d.n0 - 1), t1 = i1 - (d.n1 - 1), t2 = i2 - (d.n2 - 1);
    const long long slot = (static_cast<long long>((t0 + d.P0) % d.P0) * d.P1 + (t1 + d.P1) % d.P1) * d.P2 +
                           (t2 + d.P2) % d.P2;
    dK[(c0 + c) * noff + off] = acc[c * gsz + slot].x * scale;
  }
}

// Circular mode: dKper[c, tau] = sum of dK over the linear offsets t with
// t = tau mod n (t_a in {tau_a, tau_a - n} within [-(n_a - 1), n_a - 1]).
static __global__ void k_kg_extract_periodic(const float2* __restrict__ acc, float* __restrict__ dK, KgDims d, int c0,
                                             int ncc, float scale) {
  const long long nper = static_cast<long long>(d.n0) * d.n1 * d.n2;
  const long long gsz = static_cast<long long>(d.P0) * d.P1 * d.P2;
  const long long total = nper * ncc;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long c = e / nper, off = e % nper;
    long long r = off;
    const int u2 = static_cast<int>(r % d.n2);
    r /= d.n2;
    const int u1 = static_cast<int>(r % d.n1);
    const int u0 = static_cast<int>(r / d.n1);
    float sum = 0.f;
    for (int k0 = 0; k0 < (u0 > 0 ? 2 : 1); ++k0)
      for (int k1 = 0; k1 < (u1 > 0 ? 2 : 1); ++k1)
        for (int k2 = 0; k2 < (u2 > 0 ? 2 : 1); ++k2) {
          const int t0 = u0 - k0 * d.n0, t1 = u1 - k1 * d.n1, t2 = u2 - k2 * d.n2;
          const long long slot = (static_cast<long long>((t0 + d.P0) % d.P0) * d.P1 + (t1 + d.P1) % d.P1) * d.P2 +
                                 (t2 + d.P2) % d.P2;
          sum += acc[c * gsz + slot].x;
        }
    dK[(c0 + c) * nper + off] = sum * scale;
  }
}

}  // namespace hnd2
