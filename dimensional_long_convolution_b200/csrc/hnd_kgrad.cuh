// hnd_kgrad.cuh -- the gradient with respect to the kernel values,
//   dK[c, t] = sum_b sum_{i in [0,n)^d} q[b,c,i] dy[b,c,i] u[b,c,i - t],
// t in [-(n-1), n-1]^d, u = k v: the cross-correlation of z = q dy with u,
// summed over the batch, through zero-padded transforms on the 2n grid
// (blog "Native multi-dimensional subquadratic operators via input-dependent
// long convolutions", gradient sections: the kernel gradient by correlation).
//   k_kg_pad      w = u + i z (both real) zero-padded into one complex grid
//                 per volume [vol][P^d]
//   (axis transforms of hnd_filter2.cuh, zero pencils skipped)
//   k_kg_corr     with W the transform of w and Wm = W[-k]:
//                   U = (W + conj Wm) / 2,  Z = (W - conj Wm) / (2i),
//                   Z conj(U) = Im(W Wm) / 2 - i (|W|^2 - |Wm|^2) / 4,
//                 A_c = sum_b Z_b conj(U_b), b in order (deterministic); two
//                 channels share one grid: acc = conj(A_c1) - i conj(A_c2)
//   (axis transforms again: F(conj(A1 + i A2)) = conj(IDFT(A1) + i IDFT(A2))
//    and both inverses are real, so the result is dK_c1 - i dK_c2, unnormalised)
//   k_kg_extract  dK[c, t] = (Re or -Im)(acc)[t mod P] / prod P
// Axes are scalars (an unused axis has extent 1).  For the long 1D tier the
// grids are in the split order of hnd_long1d.cuh, whose frequency negation
// k -> P - k is taken digit by digit with borrows.
#pragma once

#include "hnd_fused2.cuh"

namespace hnd2 {

struct KgDims {
  int n0, n1, n2;       // grid (1 for unused axes)
  int P0, P1, P2;       // padded grid (1 for unused axes)
  int l0, l1, l2;       // log2 of P0, P1, P2 (all powers of two)
};

template <class T>
static __global__ void k_kg_pad(const T* __restrict__ k, const T* __restrict__ v, const T* __restrict__ q,
                                const T* __restrict__ dy, float2* __restrict__ grid, KgDims d, int B, int C, int c0,
                                int nvol) {
  const int lg = d.l0 + d.l1 + d.l2;          // log2 of the grid size
  const long long L = static_cast<long long>(d.n0) * d.n1 * d.n2;
  const long long total = static_cast<long long>(nvol) << lg;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int vv = static_cast<int>(e >> lg);
    const unsigned r = static_cast<unsigned>(e & ((1LL << lg) - 1));     // grids are below 2^32 points
    const int s2 = static_cast<int>(r & (d.P2 - 1));
    const int s1 = static_cast<int>((r >> d.l2) & (d.P1 - 1));
    const int s0 = static_cast<int>(r >> (d.l1 + d.l2));
    float2 val = make_float2(0.f, 0.f);
    if (s0 < d.n0 && s1 < d.n1 && s2 < d.n2) {
      const int cl = vv / B, bb = vv % B;
      const long long idx = (static_cast<long long>(bb) * C + c0 + cl) * L + (static_cast<long long>(s0) * d.n1 + s1) * d.n2 + s2;
      val = make_float2(Act<T>::ld_g(k + idx) * Act<T>::ld_g(v + idx), Act<T>::ld_g(q + idx) * Act<T>::ld_g(dy + idx));
    }
    (*HND_G(&grid[e])) = val;
  }
}

// Position of -k for the frequency at position r: per axis (P_a - k_a) mod P_a
// on the natural grid; on the long 1D split order (split0 > 0: factors
// split0, split1, split2) the digits of P - k with borrows.
__device__ __forceinline__ long long kg_neg(long long r, const KgDims& d, int split0, int split1, int split2) {
  if (split0 == 0) {
    const unsigned ru = static_cast<unsigned>(r);
    const unsigned k2 = ru & (d.P2 - 1), k1 = (ru >> d.l2) & (d.P1 - 1), k0 = ru >> (d.l1 + d.l2);
    const unsigned m0 = (d.P0 - k0) & (d.P0 - 1), m1 = (d.P1 - k1) & (d.P1 - 1), m2 = (d.P2 - k2) & (d.P2 - 1);
    return static_cast<long long>((((m0 << d.l1) | m1) << d.l2) | m2);
  }
  // r = (k0 P1 + k1) P2 + k2 holds X(k0 + P0 k1 + P0 P1 k2)
  const int k2 = static_cast<int>(r % split2);
  const long long r1 = r / split2;
  const int k1 = static_cast<int>(r1 % split1);
  const int k0 = static_cast<int>(r1 / split1);
  int m0, m1, m2;
  if (k0 != 0) {
    m0 = split0 - k0, m1 = split1 - 1 - k1, m2 = split2 - 1 - k2;
  } else if (k1 != 0) {
    m0 = 0, m1 = split1 - k1, m2 = split2 - 1 - k2;
  } else {
    m0 = 0, m1 = 0, m2 = (split2 - k2) % split2;
  }
  return (static_cast<long long>(m0) * split1 + m1) * split2 + m2;
}

// gw: [ncc B][P^d] transformed grids (channel-major, sample-minor);
// acc: [(ncc + 1) / 2][P^d], channels 2h and 2h + 1 in grid h.
static __global__ void k_kg_corr(const float2* __restrict__ gw, float2* __restrict__ acc, KgDims d, int B, int ncc,
                                 long long gsz, int split0, int split1, int split2) {
  const int nh = (ncc + 1) / 2;
  const int lg = d.l0 + d.l1 + d.l2;
  const long long total = gsz * nh;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long h = e >> lg, r = e & (gsz - 1);
    const long long rn = kg_neg(r, d, split0, split1, split2);
    float are[2] = {0.f, 0.f}, aim[2] = {0.f, 0.f};
    for (int j = 0; j < 2; ++j) {
      const long long c = 2 * h + j;
      if (c >= ncc) break;
      for (int b = 0; b < B; ++b) {
        const long long o = (c * B + b) * gsz;
        const float2 w = (*HND_G(&gw[o + r])), wm = (*HND_G(&gw[o + rn]));
        are[j] += 0.5f * (w.x * wm.y + w.y * wm.x);                                  // Im(W Wm) / 2
        aim[j] -= 0.25f * ((w.x * w.x + w.y * w.y) - (wm.x * wm.x + wm.y * wm.y));   // -(|W|^2 - |Wm|^2) / 4
      }
    }
    // conj(A1) - i conj(A2) = (a1r - a2i) + i (-a1i - a2r)
    (*HND_G(&acc[e])) = make_float2(are[0] - aim[1], -aim[0] - are[1]);
  }
}

// channel c of the chunk sits in grid c / 2: even c the real part, odd c
// minus the imaginary part
__device__ __forceinline__ float kg_part(const float2* acc, long long c, long long gsz, long long slot) {
  const float2 x = (*HND_G(&acc[(c >> 1) * gsz + slot]));
  return (c & 1) ? -x.y : x.x;
}

static __global__ void k_kg_extract(const float2* __restrict__ acc, float* __restrict__ dK, KgDims d, int c0, int ncc,
                                    float scale) {
  // a chunk's outputs are fewer than 2^31 (at most one grid per channel of
  // the chunk budget), so the index arithmetic stays in 32 bits
  const unsigned E0 = 2 * d.n0 - 1, E1 = 2 * d.n1 - 1, E2 = 2 * d.n2 - 1;
  const unsigned noff = E0 * E1 * E2;
  const long long gsz = static_cast<long long>(d.P0) * d.P1 * d.P2;
  const unsigned total = noff * static_cast<unsigned>(ncc);
  for (unsigned e = blockIdx.x * blockDim.x + threadIdx.x; e < total; e += gridDim.x * blockDim.x) {
    const unsigned c = e / noff, off = e - c * noff;
    const unsigned i2 = off % E2, r = off / E2;
    const unsigned i1 = r % E1, i0 = r / E1;
    const int t0 = static_cast<int>(i0) - (d.n0 - 1), t1 = static_cast<int>(i1) - (d.n1 - 1),
              t2 = static_cast<int>(i2) - (d.n2 - 1);
    const unsigned slot = ((static_cast<unsigned>(t0 + d.P0) & (d.P0 - 1)) << (d.l1 + d.l2)) |
                          ((static_cast<unsigned>(t1 + d.P1) & (d.P1 - 1)) << d.l2) |
                          (static_cast<unsigned>(t2 + d.P2) & (d.P2 - 1));
    (*HND_G(&dK[static_cast<long long>(c0 + c) * noff + off])) = kg_part(acc, c, gsz, slot) * scale;
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
          sum += kg_part(acc, c, gsz, slot);
        }
    (*HND_G(&dK[(c0 + c) * nper + off])) = sum * scale;
  }
}

}  // namespace hnd2
