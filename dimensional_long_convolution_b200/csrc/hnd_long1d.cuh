// hnd_long1d.cuh -- 1D grids longer than one transform pencil (n in
// [512, 2^26]): the zero-padded length-P transform (P = 2n) as a multi-level
// split P = P0 P1 (P2) with every factor at most 512, on the row-major view
// [P0][P1][P2] of each volume's grid (j = (j0 P1 + j1) P2 + j2):
//   forward   transform along axis 0 (the padded half j0 >= P0/2 is zero),
//             twiddle W_P^{k0 r} (r the flattened later index), then the same
//             split recursively on the later axes
//             -> X(k0 + P0 k1 + P0 P1 k2) at [k0][k1][k2] (the spectrum is kept
//             in this order)
//   modulate  Y = X S (or X conj(S) for the adjoint), stored conjugated
//   inverse   the same steps in reverse order (last axis first, each twiddle
//             after the transform of its level's later axes): every step is
//             a symmetric operator, so the reversed chain applied to data in
//             split order is the DFT in natural order; on conjugated data it
//             gives the conjugate of the unnormalised inverse at i = j
//   output    y[i] = q[i] Re(.) for i < n (the crop), optional second gate
// (HyenaND pages: arXiv 2607.19378 summary, d = 1 long context through the
// zero-padded FFT path; blog "Native multi-dimensional subquadratic operators
// via input-dependent long convolutions", section "HyenaND".)
// The axis transforms are k_fft_axis2 of hnd_filter2.cuh.
#pragma once

#include "hnd_fused2.cuh"

namespace hnd2 {

// zero-padded a . b of volumes [v0, v0 + nvol) (memory order b C + c)
template <class T>
static __global__ void k_l1_pad(const T* __restrict__ a, const T* __restrict__ b, float2* __restrict__ grid, int n,
                                long long P, long long v0, int nvol) {
  const long long total = P * nvol;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long v = e / P, j = e % P;
    float val = 0.f;
    if (j < n) {
      const long long o = (v0 + v) * n + j;
      val = Act<T>::ld_g(a + o) * Act<T>::ld_g(b + o);
    }
    grid[e] = make_float2(val, 0.f);
  }
}

// Twiddle of level a of the split: on the view [..][P_a][R] (R = Q / P_a the
// points of the later levels, Q = P_a R), element (k, r) *= W_Q^{k r},
// W_Q = exp(-2 pi i / Q).  k r < Q, and Q is a power of two, so the angle is
// the float ratio of two integers (exact while k r < 2^24).
static __global__ void k_l1_twiddle(float2* __restrict__ grid, int Pa, long long Q, long long total) {
  const long long R = Q / Pa;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long m = ((e / R) % Pa) * (e % R);
    float s, c;
    sincospif(-2.f * (static_cast<float>(m) / static_cast<float>(Q)), &s, &c);
    const float2 x = grid[e];
    grid[e] = make_float2(x.x * c - x.y * s, x.x * s + x.y * c);
  }
}

// grid = conj(grid S_c) with S_c (or conj S_c when sconj < 0) of the volume's
// channel and sample; spec: [C][P] per sample set, sample stride sbs (complex)
static __global__ void k_l1_modulate(float2* __restrict__ grid, const float2* __restrict__ spec, long long sbs,
                                     float sconj, long long P, int C, long long v0, int nvol) {
  const long long total = P * nvol;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long v = v0 + e / P, r = e % P;
    const long long b = v / C, c = v % C;
    const float2 S = __ldg(spec + b * sbs + c * P + r);
    const float si = sconj * S.y;
    const float2 x = grid[e];
    grid[e] = make_float2(x.x * S.x - x.y * si, -(x.x * si + x.y * S.x));
  }
}

template <class T, bool DUAL>
static __global__ void k_l1_out(const float2* __restrict__ grid, const T* __restrict__ q, T* __restrict__ y,
                                const T* __restrict__ g2, T* __restrict__ y2, int n, long long P, long long v0,
                                int nvol) {
  const long long total = static_cast<long long>(n) * nvol;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long v = e / n, i = e % n;
    const float r = grid[v * P + i].x;
    const long long o = (v0 + v) * n + i;
    Act<T>::st_g(y + o, r * Act<T>::ld_g(q + o));
    if constexpr (DUAL) Act<T>::st_g(y2 + o, r * Act<T>::ld_g(g2 + o));
  }
}

// filter grids (after the forward four-step) -> spectrum [c0 + c][P], scaled
static __global__ void k_l1_spec_store(const float2* __restrict__ grid, float2* __restrict__ spec, long long P, int c0,
                                       int nc, float scale) {
  const long long total = P * nc;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float2 x = grid[e];
    spec[static_cast<long long>(c0) * P + e] = make_float2(x.x * scale, x.y * scale);
  }
}

// library order [C][P0][P1][P2] (X(k0 + P0 k1 + P0 P1 k2) at (k0 P1 + k1) P2 + k2;
// P2 = 1 for a two-level split) <-> natural half spectrum [C][n + 1]; the
// import fills the other half by Hermitian symmetry
static __device__ __forceinline__ long long l1_pos(long long k, int P0, int P1, int P2) {
  return ((k % P0) * P1 + (k / P0) % P1) * P2 + k / (static_cast<long long>(P0) * P1);
}

static __global__ void k_l1_spec_export(const float2* __restrict__ lib, float2* __restrict__ nat, int n, int P0,
                                        int P1, int P2, long long C) {
  const long long P = static_cast<long long>(P0) * P1 * P2, H = n + 1LL;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < H * C;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long c = e / H, k = e % H;
    nat[e] = lib[c * P + l1_pos(k, P0, P1, P2)];
  }
}

static __global__ void k_l1_spec_import(const float2* __restrict__ nat, float2* __restrict__ lib, int n, int P0,
                                        int P1, int P2, long long C, long long pitch, float scale) {
  const long long P = static_cast<long long>(P0) * P1 * P2;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < P * C;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long c = e / P, r = e % P;
    const long long k = r / (static_cast<long long>(P1) * P2) + P0 * ((r / P2) % P1) +
                        static_cast<long long>(P0) * P1 * (r % P2);
    float2 s;
    if (k <= n) {
      s = nat[c * pitch + k];
    } else {
      s = nat[c * pitch + (P - k)];
      s.y = -s.y;
    }
    lib[e] = make_float2(s.x * scale, s.y * scale);
  }
}

}  // namespace hnd2
