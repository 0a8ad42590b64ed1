// hnd_long1d.cuh -- 1D grids longer than one transform pencil (n in
// [512, 131072]): the zero-padded length-P transform (P = 2n) as a four-step
// factorisation P = P0 P1 on the [P0][P1] view of each volume's grid
// (j = P1 j0 + j1):
//   forward   transform along j0 (the padded half: j0 >= P0/2 is zero),
//             twiddle W_P^{k0 j1}, transform along j1
//             -> X(k0 + P0 k1) at [k0][k1] (the spectrum is kept in this order)
//   modulate  Y = X S (or X conj(S) for the adjoint), stored conjugated
//   inverse   transform along k1, twiddle W_P^{k0 i1}, transform along k0:
//             the conjugate of the unnormalised inverse at i = P1 i0 + i1
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

// grid[g][r0][r1] *= W_P^{r0 r1} (W_P = exp(-2 pi i / P)), P = P0 P1
static __global__ void k_l1_twiddle(float2* __restrict__ grid, int P0, int P1, long long ngrids) {
  const long long P = static_cast<long long>(P0) * P1;
  const long long total = P * ngrids;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = e % P;
    const long long m = ((r / P1) * (r % P1)) % P;
    float s, c;
    sincospif(-2.f * (static_cast<float>(m) / static_cast<float>(P)), &s, &c);   // exact ratio: P is 2^k
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

// library order [C][P0][P1] (X(k0 + P0 k1) at k0 P1 + k1) <-> natural half
// spectrum [C][n + 1]; the import fills the other half by Hermitian symmetry
static __global__ void k_l1_spec_export(const float2* __restrict__ lib, float2* __restrict__ nat, int n, int P0,
                                        int P1, long long C) {
  const long long P = static_cast<long long>(P0) * P1, H = n + 1;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < H * C;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long c = e / H, k = e % H;
    nat[e] = lib[c * P + (k % P0) * P1 + k / P0];
  }
}

static __global__ void k_l1_spec_import(const float2* __restrict__ nat, float2* __restrict__ lib, int n, int P0,
                                        int P1, long long C, long long pitch, float scale) {
  const long long P = static_cast<long long>(P0) * P1;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < P * C;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long c = e / P, r = e % P;
    const long long k = (r / P1) + static_cast<long long>(P0) * (r % P1);
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
