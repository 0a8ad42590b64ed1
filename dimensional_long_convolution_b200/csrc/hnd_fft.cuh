// hnd_fft.cuh -- register/shared-memory FFT building blocks for the padded
// (linear) FFT convolution of the HyenaND pages (blog section "nSubQ": forward
// FFT, pointwise product in frequency space, inverse FFT; arXiv 2607.19378
// summary, "Methodologie": zero padding to twice the grid).
//
// Building block: a length-2N transform of a pencil whose last N inputs are
// zero (zero padding), computed as two length-N transforms:
//   X[2m]   = FFT_N(x)[m]
//   X[2m+1] = FFT_N(x * W_2N^j)[m]
// and the matching inverse that keeps only the first N outputs:
//   y[i]    = IFFT_N(Y_even)[i] + W_2N^-i * IFFT_N(Y_odd)[i],   i < N.
// The two halves ("paths") run side by side in the same threads.
//
// A pencil is owned by G = N/8 consecutive lanes of one warp; each lane holds
// 8 complex values per path in registers.  The length-N FFT is a Stockham
// radix-8 (+ a final radix-2/4) decomposition; between passes the lanes trade
// values through a small padded shared-memory buffer (one float4 = both paths
// per index).  Layouts:
//   natural layout  (forward input, inverse output):  slot s  <->  g + s*G
//   spectral layout (forward output, inverse input):  slot s  <->  f(g, s)
// with f defined by spec_index<N>().  The spectral layout is never reordered
// into natural frequency order: the channel spectrum is stored in the same
// order, so the pointwise product needs no bit reversal.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "hnd_bounds.cuh"

namespace hnd {

constexpr int kTab = 512;   // twiddle table: W_512^e, e in [0, 512)

// ----------------------------------------------------------------- complex
__device__ __forceinline__ float2 c_add(float2 a, float2 b) { return make_float2(a.x + b.x, a.y + b.y); }
__device__ __forceinline__ float2 c_sub(float2 a, float2 b) { return make_float2(a.x - b.x, a.y - b.y); }
__device__ __forceinline__ float2 c_mul(float2 a, float2 b) {
  return make_float2(fmaf(a.x, b.x, -a.y * b.y), fmaf(a.x, b.y, a.y * b.x));
}
// a * conj(b)
__device__ __forceinline__ float2 c_mulc(float2 a, float2 b) {
  return make_float2(fmaf(a.x, b.x, a.y * b.y), fmaf(a.y, b.x, -a.x * b.y));
}
__device__ __forceinline__ float2 c_conj(float2 a) { return make_float2(a.x, -a.y); }
__device__ __forceinline__ float2 c_scale(float2 a, float s) { return make_float2(a.x * s, a.y * s); }
template <bool INV>
__device__ __forceinline__ float2 c_tw(float2 a, float2 w) { return INV ? c_mulc(a, w) : c_mul(a, w); }
// multiply by -i (forward) or +i (inverse)
template <bool INV>
__device__ __forceinline__ float2 c_rot(float2 a) { return INV ? make_float2(-a.y, a.x) : make_float2(a.y, -a.x); }

// ------------------------------------------------------------ small DFTs
template <bool INV>
__device__ __forceinline__ void dft2(float2& a0, float2& a1) {
  const float2 t = c_sub(a0, a1);
  a0 = c_add(a0, a1);
  a1 = t;
}

template <bool INV>
__device__ __forceinline__ void dft4(float2& a0, float2& a1, float2& a2, float2& a3) {
  const float2 c0 = c_add(a0, a2), c2 = c_sub(a0, a2);
  const float2 c1 = c_add(a1, a3), c3 = c_rot<INV>(c_sub(a1, a3));
  a0 = c_add(c0, c1);
  a2 = c_sub(c0, c1);
  a1 = c_add(c2, c3);
  a3 = c_sub(c2, c3);
}

// Natural-order DFT of 8 points (radix-2 split into two DFT4).
template <bool INV>
__device__ __forceinline__ void dft8(float2* a) {
  const float h = 0.70710678118654752440f;
  float2 b0 = c_add(a[0], a[4]), b4 = c_sub(a[0], a[4]);
  float2 b1 = c_add(a[1], a[5]), b5 = c_sub(a[1], a[5]);
  float2 b2 = c_add(a[2], a[6]), b6 = c_sub(a[2], a[6]);
  float2 b3 = c_add(a[3], a[7]), b7 = c_sub(a[3], a[7]);
  // b5 *= W8^1, b6 *= W8^2, b7 *= W8^3 with W8 = exp(-+ i pi / 4)
  b6 = c_rot<INV>(b6);
  if (INV) {
    b5 = make_float2((b5.x - b5.y) * h, (b5.x + b5.y) * h);
    b7 = make_float2((-b7.x - b7.y) * h, (b7.x - b7.y) * h);
  } else {
    b5 = make_float2((b5.x + b5.y) * h, (b5.y - b5.x) * h);
    b7 = make_float2((b7.y - b7.x) * h, (-b7.x - b7.y) * h);
  }
  dft4<INV>(b0, b1, b2, b3);
  dft4<INV>(b4, b5, b6, b7);
  a[0] = b0; a[2] = b1; a[4] = b2; a[6] = b3;
  a[1] = b4; a[3] = b5; a[5] = b6; a[7] = b7;
}

// ------------------------------------------------------------------- plan
// Radix sequence of a length-N FFT (N = 8 .. 512, power of two).
template <int N>
struct Plan {
  static_assert(N >= 8 && N <= 512 && (N & (N - 1)) == 0, "unsupported FFT length");
  static constexpr int G = N / 8;                       // lanes per pencil
  static constexpr int NP = (N == 8) ? 1 : (N <= 64 ? 2 : 3);
  __host__ __device__ static constexpr int R(int p) {
    return p == 0 ? 8
         : p == 1 ? (N == 16 ? 2 : N == 32 ? 4 : 8)
                  : (N == 128 ? 2 : N == 256 ? 4 : 8);
  }
  static constexpr int RL = R(NP - 1);                  // last forward radix
};

// Frequency index held in slot s of lane g after a forward transform.
template <int N>
__host__ __device__ __forceinline__ int spec_index(int g, int s) {
  constexpr int G = Plan<N>::G, RL = Plan<N>::RL;
  return g + G * (s / RL) + (s % RL) * (N / RL);
}

// Padded index inside a pencil's exchange buffer (one pad slot every 8).
__host__ __device__ __forceinline__ int xpad(int i) { return i + (i >> 3); }
template <int N>
struct XBuf { static constexpr int kFloat4 = N + N / 8; };  // float4 per pencil

// Lane mask of the G lanes that own one pencil.
template <int N>
__device__ __forceinline__ unsigned pencil_mask(int lane) {
  constexpr int G = Plan<N>::G;
  if constexpr (G >= 32) {
    return 0xffffffffu;
  } else {
    const unsigned m = (1u << G) - 1u;
    return m << ((lane / G) * G);
  }
}

// One Stockham pass of radix RP over both paths.  Slot b*RP + r holds the
// input index j + r*N/RP (j = g + G*b) on entry and the output index
// (j/NS)*NS*RP + j%NS + r*NS on exit.
template <int N, int RP, int NS, bool INV>
__device__ __forceinline__ void pass2(float2 (&x)[2][8], int g, const float2* __restrict__ T) {
  constexpr int G = Plan<N>::G;
#pragma unroll
  for (int b = 0; b < 8 / RP; ++b) {
    if constexpr (NS > 1) {
      const int jm = (g + G * b) & (NS - 1);
#pragma unroll
      for (int r = 1; r < RP; ++r) {
        const float2 w = (*HND_S(&T[(jm * r) * (kTab / (NS * RP))]));
        x[0][b * RP + r] = c_tw<INV>(x[0][b * RP + r], w);
        x[1][b * RP + r] = c_tw<INV>(x[1][b * RP + r], w);
      }
    }
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      if constexpr (RP == 8) dft8<INV>(&x[p][b * 8]);
      else if constexpr (RP == 4) dft4<INV>(x[p][b * 4], x[p][b * 4 + 1], x[p][b * 4 + 2], x[p][b * 4 + 3]);
      else dft2<INV>(x[p][b * 2], x[p][b * 2 + 1]);
    }
  }
}

// Trade values between passes: write the outputs of a (RPO, NSO) pass, read
// the inputs of a radix-RPI pass.
template <int N, int RPO, int NSO, int RPI>
__device__ __forceinline__ void exch2(float2 (&x)[2][8], int g, float4* buf, unsigned mask) {
  constexpr int G = Plan<N>::G;
  __syncwarp(mask);
#pragma unroll
  for (int b = 0; b < 8 / RPO; ++b) {
    const int j = g + G * b;
    const int base = (j / NSO) * NSO * RPO + (j % NSO);
#pragma unroll
    for (int r = 0; r < RPO; ++r) {
      const int s = b * RPO + r;
      (*HND_S(&buf[xpad(base + r * NSO)])) = make_float4(x[0][s].x, x[0][s].y, x[1][s].x, x[1][s].y);
    }
  }
  __syncwarp(mask);
#pragma unroll
  for (int b = 0; b < 8 / RPI; ++b) {
    const int j = g + G * b;
#pragma unroll
    for (int r = 0; r < RPI; ++r) {
      const int s = b * RPI + r;
      const float4 t = (*HND_S(&buf[xpad(j + r * (N / RPI))]));
      x[0][s] = make_float2(t.x, t.y);
      x[1][s] = make_float2(t.z, t.w);
    }
  }
}

// Length-N FFT of both paths.  Forward: natural -> spectral layout.
// Inverse (unnormalised, conjugate twiddles): spectral -> natural layout.
template <int N, bool INV>
__device__ __forceinline__ void fft2(float2 (&x)[2][8], int g, float4* buf, const float2* T, unsigned mask) {
  using PL = Plan<N>;
  if constexpr (!INV) {
    constexpr int R0 = PL::R(0);
    pass2<N, R0, 1, false>(x, g, T);
    if constexpr (PL::NP >= 2) {
      constexpr int R1 = PL::R(1);
      exch2<N, R0, 1, R1>(x, g, buf, mask);
      pass2<N, R1, R0, false>(x, g, T);
      if constexpr (PL::NP >= 3) {
        constexpr int R2 = PL::R(2);
        exch2<N, R1, R0, R2>(x, g, buf, mask);
        pass2<N, R2, R0 * R1, false>(x, g, T);
      }
    }
  } else {
    constexpr int Q0 = PL::R(PL::NP - 1);
    pass2<N, Q0, 1, true>(x, g, T);
    if constexpr (PL::NP >= 2) {
      constexpr int Q1 = PL::R(PL::NP - 2 >= 0 ? PL::NP - 2 : 0);
      exch2<N, Q0, 1, Q1>(x, g, buf, mask);
      pass2<N, Q1, Q0, true>(x, g, T);
      if constexpr (PL::NP >= 3) {
        constexpr int Q2 = PL::R(0);
        exch2<N, Q1, Q0, Q2>(x, g, buf, mask);
        pass2<N, Q2, Q0 * Q1, true>(x, g, T);
      }
    }
  }
}

// Zero-padded forward transform of length 2N.  On entry x[0][s] = z[g + s*G]
// (the N non-zero inputs).  On exit x[p][s] = Z[2 * spec_index(g, s) + p].
template <int N>
__device__ __forceinline__ void padded_fwd(float2 (&x)[2][8], int g, float4* buf, const float2* T, unsigned mask) {
  constexpr int G = Plan<N>::G;
#pragma unroll
  for (int s = 0; s < 8; ++s) x[1][s] = c_mul(x[0][s], (*HND_S(&T[(g + s * G) * (kTab / (2 * N))])));
  fft2<N, false>(x, g, buf, T, mask);
}

// Inverse of length 2N keeping outputs [0, N).  On entry x[p][s] =
// Y[2 * spec_index(g, s) + p]; on exit x[0][s] = y[g + s*G] (unnormalised).
template <int N>
__device__ __forceinline__ void padded_inv(float2 (&x)[2][8], int g, float4* buf, const float2* T, unsigned mask) {
  constexpr int G = Plan<N>::G;
  fft2<N, true>(x, g, buf, T, mask);
#pragma unroll
  for (int s = 0; s < 8; ++s) x[0][s] = c_add(x[0][s], c_mulc(x[1][s], (*HND_S(&T[(g + s * G) * (kTab / (2 * N))]))));
}

// Natural index of the partner frequency -k (mod 2N) of spectral slot (f, p):
// even path f -> (N - f) mod N, odd path f -> N - 1 - f.
template <int N>
__device__ __forceinline__ int partner_even(int f) { return (N - f) & (N - 1); }
template <int N>
__device__ __forceinline__ int partner_odd(int f) { return N - 1 - f; }

// After a forward transform: fetch Z[-k] for every held Z[k] through the
// pencil's exchange buffer (indexed by natural half-frequency f).
template <int N>
__device__ __forceinline__ void fetch_partner(const float2 (&x)[2][8], float2 (&xp)[2][8], int g, float4* buf,
                                              unsigned mask) {
  __syncwarp(mask);
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const int f = spec_index<N>(g, s);
    (*HND_S(&buf[xpad(f)])) = make_float4(x[0][s].x, x[0][s].y, x[1][s].x, x[1][s].y);
  }
  __syncwarp(mask);
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const int f = spec_index<N>(g, s);
    const float4 te = (*HND_S(&buf[xpad(partner_even<N>(f))]));
    const float4 to = (*HND_S(&buf[xpad(partner_odd<N>(f))]));
    xp[0][s] = make_float2(te.x, te.y);
    xp[1][s] = make_float2(to.z, to.w);
  }
}

// ------------------------------------------------------------ activations
struct IOF32 {
  using T = float;
  static __device__ __forceinline__ float ld(const float* p) { return __ldcs(HND_G(p)); }
  static __device__ __forceinline__ void st(float* p, float x) { __stcs(HND_G(p), x); }
};
struct IOBF16 {
  using T = __nv_bfloat16;
  static __device__ __forceinline__ float ld(const __nv_bfloat16* p) {
    const unsigned short b = __ldcs(HND_G(reinterpret_cast<const unsigned short*>(p)));
    return __uint_as_float(static_cast<unsigned>(b) << 16);
  }
  static __device__ __forceinline__ void st(__nv_bfloat16* p, float x) {
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    __stcs(HND_G(reinterpret_cast<unsigned short*>(p)), *reinterpret_cast<const unsigned short*>(&h));
  }
};

// Row-pair packing (two real rows a, b in one complex transform):
// X_a = (Z[k] + conj Z[-k]) / 2,  X_b = (Z[k] - conj Z[-k]) / (2i).
__device__ __forceinline__ float2 unpack_a(float2 z, float2 zm) {
  return make_float2(0.5f * (z.x + zm.x), 0.5f * (z.y - zm.y));
}
__device__ __forceinline__ float2 unpack_b(float2 z, float2 zm) {
  return make_float2(0.5f * (z.y + zm.y), 0.5f * (zm.x - z.x));
}
// W[k] = Y_a + i Y_b, W[-k] = conj(Y_a) + i conj(Y_b)
__device__ __forceinline__ float2 pack_pos(float2 ya, float2 yb) { return make_float2(ya.x - yb.y, ya.y + yb.x); }
__device__ __forceinline__ float2 pack_neg(float2 ya, float2 yb) { return make_float2(ya.x + yb.y, yb.x - ya.y); }

// Device status word (first 16 bytes of the workspace).
__device__ __forceinline__ void set_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

}  // namespace hnd
