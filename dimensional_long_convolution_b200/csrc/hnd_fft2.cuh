// hnd_fft2.cuh -- packed two-path FFT core for sm_100a.
//
// The zero-padded length-2N transform of a pencil whose last N inputs are 0
// (HyenaND pages: zero padding to twice the grid gives the linear
// convolution) splits into two length-N transforms that share every twiddle:
//   X[2m]   = FFT_N(x)[m]                (path 0)
//   X[2m+1] = FFT_N(x W_2N^j)[m]         (path 1)
// and the inverse that keeps outputs [0, N):
//   y[i]    = IFFT_N(Y0)[i] + W_2N^-i IFFT_N(Y1)[i].
// Both paths live in the two lanes of float2 registers ("cp": re = (path0.re,
// path1.re), im = (path0.im, path1.im)), so every butterfly is one packed
// FADD2/FFMA2 for both paths: the fp32 work is unchanged, the issue slots
// halve.
//
// A length-N transform (N = R1 * R2, R1 = 8) is owned by G = R2 lanes; each
// lane holds R1 slots.  Pass 1 is a radix-R1 DFT on x[g + r G]; the lanes
// trade values once through a swizzled shared buffer; pass 2 is a radix-R2
// DFT with twiddles W_N^{j r}.  Layouts:
//   natural  (forward input, inverse output):  slot s <-> index g + s G
//   spectral (forward output, inverse input):  slot s <-> g + G (s / R2) + (s % R2) R1
// The spectral order is never reordered: the channel spectrum is stored in
// it, so the pointwise product needs no bit reversal.
#pragma once

#include <type_traits>

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "hnd_bounds.cuh"

namespace hnd2 {

// Programmatic dependent launch: the stage kernels run back to back on one
// stream.  Each lets the next stage's CTAs be scheduled as soon as all of its
// own CTAs have started (they then build their tables on SMs freed by this
// stage's tail), and waits for the previous grid to complete, with its
// memory visible, before its first global access.  Both are no-ops for a
// launch without the programmatic-serialization attribute.
__device__ __forceinline__ void pdl_release() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ------------------------------------------------------------ packed fp32
__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }
__device__ __forceinline__ float2 padd(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 psub(float2 a, float2 b) { return __fadd2_rn(a, make_float2(-b.x, -b.y)); }
__device__ __forceinline__ float2 pmul(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 pfma(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

struct cp {
  float2 re, im;
};
__device__ __forceinline__ cp cadd(cp a, cp b) { return {padd(a.re, b.re), padd(a.im, b.im)}; }
__device__ __forceinline__ cp csub(cp a, cp b) { return {psub(a.re, b.re), psub(a.im, b.im)}; }

// x * (c + i s) for both paths (w4 = (c, c, s, s)); INV: x * (c - i s)
template <bool INV>
__device__ __forceinline__ cp ctw(cp x, float4 w4) {
  const float2 cc = make_float2(w4.x, w4.y), ss = make_float2(w4.z, w4.w);
  const float2 nss = make_float2(-w4.z, -w4.w);
  if (INV) return {pfma(x.im, ss, pmul(x.re, cc)), pfma(x.re, nss, pmul(x.im, cc))};
  return {pfma(x.im, nss, pmul(x.re, cc)), pfma(x.re, ss, pmul(x.im, cc))};
}
// x * s with a different complex factor per path (s = (s0.re, s1.re), (s0.im, s1.im))
__device__ __forceinline__ cp cmulp(cp x, float2 sre, float2 sim) {
  const float2 nsim = make_float2(-sim.x, -sim.y);
  return {pfma(x.im, nsim, pmul(x.re, sre)), pfma(x.re, sim, pmul(x.im, sre))};
}

// ------------------------------------------------------------ small DFTs
// Natural-order DFT4 of (a0, a1, a2, a3); forward sign -i, inverse +i.
template <bool INV>
__device__ __forceinline__ void dft4(cp& a0, cp& a1, cp& a2, cp& a3) {
  const cp c0 = cadd(a0, a2), c2 = csub(a0, a2), c1 = cadd(a1, a3), d = csub(a1, a3);
  a0 = cadd(c0, c1);
  a2 = csub(c0, c1);
  if (!INV) {   // c2 -/+ i d
    a1 = {padd(c2.re, d.im), psub(c2.im, d.re)};
    a3 = {psub(c2.re, d.im), padd(c2.im, d.re)};
  } else {
    a1 = {psub(c2.re, d.im), padd(c2.im, d.re)};
    a3 = {padd(c2.re, d.im), psub(c2.im, d.re)};
  }
}

__device__ __forceinline__ void dft2(cp& a0, cp& a1) {
  const cp t = csub(a0, a1);
  a0 = cadd(a0, a1);
  a1 = t;
}

// Natural-order DFT8, 52 packed operations (the 1/sqrt2 factors ride in FMAs).
template <bool INV>
__device__ __forceinline__ void dft8(cp* a) {
  const float2 h = f2(0.70710678118654752440f), nh = f2(-0.70710678118654752440f);
  cp b0 = cadd(a[0], a[4]), b4 = csub(a[0], a[4]);
  cp b1 = cadd(a[1], a[5]), b5 = csub(a[1], a[5]);
  cp b2 = cadd(a[2], a[6]), b6 = csub(a[2], a[6]);
  cp b3 = cadd(a[3], a[7]), b7 = csub(a[3], a[7]);
  dft4<INV>(b0, b1, b2, b3);                // even outputs 0, 2, 4, 6
  cp c0, c2;
  float2 u1, u2, u3, u4;                   // odd half: b5 W8, b6 W8^2, b7 W8^3 folded in
  if (!INV) {
    c0 = {padd(b4.re, b6.im), psub(b4.im, b6.re)};          // b4 + (-i) b6
    c2 = {psub(b4.re, b6.im), padd(b4.im, b6.re)};
    const float2 s5 = padd(b5.re, b5.im), t5 = psub(b5.im, b5.re);
    const float2 s7 = padd(b7.re, b7.im), t7 = psub(b7.im, b7.re);
    u1 = padd(s5, t7);
    u2 = psub(t5, s7);      // c1 = h (u1, u2)
    u3 = psub(s5, t7);
    u4 = padd(t5, s7);      // d  = h (u3, u4)
    a[0] = b0; a[2] = b1; a[4] = b2; a[6] = b3;
    a[1] = {pfma(h, u1, c0.re), pfma(h, u2, c0.im)};
    a[5] = {pfma(nh, u1, c0.re), pfma(nh, u2, c0.im)};
    a[3] = {pfma(h, u4, c2.re), pfma(nh, u3, c2.im)};       // c2 + (-i) d
    a[7] = {pfma(nh, u4, c2.re), pfma(h, u3, c2.im)};
  } else {
    c0 = {psub(b4.re, b6.im), padd(b4.im, b6.re)};          // b4 + (+i) b6
    c2 = {padd(b4.re, b6.im), psub(b4.im, b6.re)};
    // b5 (1 + i) h, b7 (-1 + i) h
    const float2 s5 = psub(b5.re, b5.im), t5 = padd(b5.re, b5.im);
    const float2 s7 = padd(b7.re, b7.im), t7 = psub(b7.re, b7.im);
    // p1 = h (s5, t5); p3 = h (-s7, t7)
    u1 = psub(s5, s7);
    u2 = padd(t5, t7);      // c1 = p1 + p3
    u3 = padd(s5, s7);
    u4 = psub(t5, t7);      // d  = p1 - p3
    a[0] = b0; a[2] = b1; a[4] = b2; a[6] = b3;
    a[1] = {pfma(h, u1, c0.re), pfma(h, u2, c0.im)};
    a[5] = {pfma(nh, u1, c0.re), pfma(nh, u2, c0.im)};
    a[3] = {pfma(nh, u4, c2.re), pfma(h, u3, c2.im)};       // c2 + (+i) d
    a[7] = {pfma(h, u4, c2.re), pfma(nh, u3, c2.im)};
  }
  // the even DFT4 left its outputs in b0..b3 = X0, X2, X4, X6 (set above)
}

// Natural-order DFT16 as 4 x 4: DFT4 over stride-4 inputs, twiddles
// W16^{r1 k1}, DFT4 across; the result is read back in natural order.
template <bool INV>
__device__ __forceinline__ void cmul_const(cp& x, float c, float sn) {
  // x * (c + i sn)
  const float2 cc = f2(c), ss = f2(sn), nss = f2(-sn);
  x = {pfma(x.im, nss, pmul(x.re, cc)), pfma(x.re, ss, pmul(x.im, cc))};
}

template <bool INV>
__device__ __forceinline__ void dft16(cp* a) {
  const float c1 = 0.92387953251128675613f, s1 = 0.38268343236508977173f, h = 0.70710678118654752440f;
  const float sg = INV ? 1.f : -1.f;      // forward W16^e = exp(-2 pi i e / 16)
#pragma unroll
  for (int r1 = 0; r1 < 4; ++r1) dft4<INV>(a[r1], a[r1 + 4], a[r1 + 8], a[r1 + 12]);
  // B[r1][k1] at a[r1 + 4 k1]; twiddles W16^{r1 k1}
  cmul_const<INV>(a[1 + 4], c1, sg * s1);            // e = 1
  cmul_const<INV>(a[2 + 4], h, sg * h);              // e = 2
  cmul_const<INV>(a[3 + 4], s1, sg * c1);            // e = 3
  cmul_const<INV>(a[1 + 8], h, sg * h);              // e = 2
  a[2 + 8] = INV ? cp{make_float2(-a[10].im.x, -a[10].im.y), a[10].re}
                 : cp{a[10].im, make_float2(-a[10].re.x, -a[10].re.y)};   // e = 4: -+i
  cmul_const<INV>(a[3 + 8], -h, sg * h);             // e = 6
  cmul_const<INV>(a[1 + 12], s1, sg * c1);           // e = 3
  cmul_const<INV>(a[2 + 12], -h, sg * h);            // e = 6
  cmul_const<INV>(a[3 + 12], -c1, -sg * s1);         // e = 9
#pragma unroll
  for (int k1 = 0; k1 < 4; ++k1) dft4<INV>(a[4 * k1], a[4 * k1 + 1], a[4 * k1 + 2], a[4 * k1 + 3]);
  // X[k1 + 4 k2] sits at a[4 k1 + k2]: transpose the 4 x 4 block
  cp t[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) t[i] = a[i];
#pragma unroll
  for (int k1 = 0; k1 < 4; ++k1)
#pragma unroll
    for (int k2 = 0; k2 < 4; ++k2) a[k1 + 4 * k2] = t[4 * k1 + k2];
}

// ------------------------------------------------------------------- plan
template <int N>
struct P2 {
  static_assert(N == 8 || N == 16 || N == 32 || N == 64 || N == 128 || N == 256, "packed core: N in 8..256");
  static constexpr int R1 = N >= 128 ? 16 : 8;     // slots per lane, pass-1 radix
  static constexpr int R2 = N / R1;                // pass-2 radix: 1 (single pass), 2, 4, 8, 16
  static constexpr int G = (N == 8) ? 1 : R2;      // lanes per pencil
  static constexpr bool TWO = N > 8;
};

template <int N>
__host__ __device__ __forceinline__ int spec_idx(int g, int s) {
  if constexpr (N == 8) {
    return s;
  } else {
    constexpr int G = P2<N>::G, R2 = P2<N>::R2, R1 = P2<N>::R1;
    return g + G * (s / R2) + (s % R2) * R1;
  }
}

// Padded float4 index inside a pencil's exchange buffer (one pad slot every
// 8): for the 8-lane phases of both passes the lanes land on distinct
// 16-byte bank groups, and with the thread's lane index folded into a base
// pointer every access is a compile-time offset.  A pencil's buffer holds
// N + N/8 float4.
__host__ __device__ __forceinline__ int swz(int i) { return i + (i >> 3); }
// pad by d: one pad slot every d entries (d = 8 or 16)
template <int D>
__host__ __device__ __forceinline__ int padx(int i) { return i + i / D; }

// Exchange-buffer float4 per pencil; the pencil stride keeps pencils that
// share an 8-lane phase (G < 8) on different bank groups.
template <int N>
struct XB {
  static constexpr int kPen = N + N / 8;                  // float4 per pencil (covers both pads)
  static constexpr int kWarp = (32 / P2<N>::G) * kPen;     // float4 per warp (all its pencils)
};
template <int N>
__device__ __forceinline__ int pkey(int) { return 0; }

template <int N>
__device__ __forceinline__ unsigned pmask(int lane) {
  constexpr int G = P2<N>::G;
  if constexpr (G >= 32) {
    return 0xffffffffu;
  } else {
    const unsigned m = (1u << G) - 1u;
    return m << ((lane / G) * G);
  }
}

// Per-size twiddle bases in shared memory (built once per CTA), [j][g]:
//   b[j G + g] = W_N^{2^j g}  (j = 0..3: u, u^2, u^4, u^8 for u = W_N^g)
//   b[4 G + g] = W_2N^g
// Every twiddle of a lane follows from these and the roots W_32^e (constant
// memory, compile-time indices):
//   pass-2 twiddle  W_N^{(g + G b) r} = u^r W_R1^{b r}   (G / N = 1 / R1)
//   inverse pass 2  W_N^{g r}         = u^r
//   twist           W_2N^{g + s G}    = W_2N^g W_{2 R1}^s
// with u^r the product of the bases of r's set bits (at most three complex
// products).
template <int N>
struct Tabs {
  static constexpr int G = P2<N>::G;
  static constexpr size_t kBytes = (8 * 5 * G + 15) / 16 * 16;
  float2* b;
};

static __constant__ float2 c_w32[32] =
#include "hnd_w32.inc"
    ;

template <int N>
__device__ __forceinline__ Tabs<N> tabs_at(unsigned char* base) {
  Tabs<N> t;
  t.b = reinterpret_cast<float2*>(base);
  return t;
}

// W_M^e from the 512-entry table W_512^k.
__device__ __forceinline__ float2 wtab(const float2* __restrict__ W512, int M, int e) {
  return W512[(e % M) * (512 / M)];
}

template <int N>
__device__ __forceinline__ void tabs_build(Tabs<N> t, const float2* __restrict__ W512) {
  constexpr int G = P2<N>::G;
  for (int e = threadIdx.x; e < 5 * G; e += blockDim.x) {
    const int j = e / G, g = e % G;
    *HND_S(&t.b[e]) = j < 4 ? wtab(W512, N, g << j) : wtab(W512, 2 * N, g);
  }
}

__device__ __forceinline__ float2 cmul1(float2 a, float2 b) {
  return make_float2(fmaf(a.x, b.x, -a.y * b.y), fmaf(a.x, b.y, a.y * b.x));
}

// u^R (1 <= R < 16): product of the bases u^{2^j} of R's set bits j >= J.
template <int R, int J = 0>
__device__ __forceinline__ float2 upow(const float2 (&u)[4]) {
  static_assert(R >= 1 && R < 16, "power range");
  if constexpr ((R >> J) == 1) return u[J];
  else if constexpr (((R >> J) & 1) == 0) return upow<R, J + 1>(u);
  else return cmul1(u[J], upow<R, J + 1>(u));
}

// x * W_32^E (E compile-time; E == 0: x)
template <int E>
__device__ __forceinline__ float2 mul_w32(float2 x) {
  if constexpr ((E & 31) == 0) return x;
  else if constexpr ((E & 31) == 8) return make_float2(x.y, -x.x);       // W_32^8 = -i
  else if constexpr ((E & 31) == 16) return make_float2(-x.x, -x.y);
  else if constexpr ((E & 31) == 24) return make_float2(-x.y, x.x);      // W_32^24 = i
  else return cmul1(x, c_w32[E & 31]);
}

template <int N>
__device__ __forceinline__ void load_bases(Tabs<N> t, int g, float2 (&u)[4]) {
  constexpr int G = P2<N>::G, R1 = P2<N>::R1;
  u[0] = *HND_S(&t.b[g]);
  u[1] = *HND_S(&t.b[G + g]);
  u[2] = *HND_S(&t.b[2 * G + g]);
  u[3] = R1 == 16 ? *HND_S(&t.b[3 * G + g]) : make_float2(1.f, 0.f);
}

__device__ __forceinline__ float4 w4of(float2 w) { return make_float4(w.x, w.x, w.y, w.y); }

// Compile-time loops (the twiddle exponents must be constants).
template <int I, int E, class F>
__device__ __forceinline__ void sfor(F&& f) {
  if constexpr (I < E) {
    f(std::integral_constant<int, I>{});
    sfor<I + 1, E>(f);
  }
}

// ------------------------------------------------------------------- FFTs
// Forward: natural -> spectral.  buf: this pencil's XB<N>::kPen float4.
// The forward exchange pads by R1, the inverse exchange by max(R2, 8): with the
// lane index in the low bits, each 8-lane phase hits distinct 16-byte bank
// groups, and every padded index stays below N + N/8.
template <int N>
__device__ __forceinline__ void fft_fwd(cp (&x)[P2<N>::R1], int g, float4* buf, int key, Tabs<N> t, unsigned mask) {
  constexpr int R1 = P2<N>::R1;
  if constexpr (R1 == 16) dft16<false>(x);
  else dft8<false>(x);
  if constexpr (P2<N>::TWO) {
    constexpr int G = P2<N>::G, R2 = P2<N>::R2;
    __syncwarp();
#pragma unroll
    for (int r = 0; r < R1; ++r)
      *HND_S(&buf[padx<R1>(g * R1 + r)]) = make_float4(x[r].re.x, x[r].re.y, x[r].im.x, x[r].im.y);
    __syncwarp();
    float2 u[4];
    load_bases<N>(t, g, u);
    sfor<0, R1 / R2>([&](auto bc) {
      constexpr int b = decltype(bc)::value;
      sfor<0, R2>([&](auto rc) {
        constexpr int r = decltype(rc)::value;
        const float4 v = *HND_S(&buf[padx<R1>(g + G * b + r * R1)]);
        cp y = {make_float2(v.x, v.y), make_float2(v.z, v.w)};
        if constexpr (r > 0) {
          // W_N^{(g + G b) r} = u^r W_R1^{b r}
          y = ctw<false>(y, w4of(mul_w32<(b * r % R1) * (32 / R1)>(upow<r>(u))));
        }
        x[b * R2 + r] = y;
      });
      if constexpr (R2 == 16) dft16<false>(&x[b * 16]);
      else if constexpr (R2 == 8) dft8<false>(&x[b * 8]);
      else if constexpr (R2 == 4) dft4<false>(x[b * 4], x[b * 4 + 1], x[b * 4 + 2], x[b * 4 + 3]);
      else dft2(x[b * 2], x[b * 2 + 1]);
    });
  }
}

// Inverse (unnormalised): spectral -> natural.
template <int N>
__device__ __forceinline__ void fft_inv(cp (&x)[P2<N>::R1], int g, float4* buf, int key, Tabs<N> t, unsigned mask) {
  constexpr int R1 = P2<N>::R1;
  if constexpr (!P2<N>::TWO) {
    dft8<true>(x);
  } else {
    constexpr int G = P2<N>::G, R2 = P2<N>::R2;
    constexpr int PD = R2 < 8 ? 8 : R2;      // pad stride; keeps the buffer within N + N/8
#pragma unroll
    for (int b = 0; b < R1 / R2; ++b) {
      if constexpr (R2 == 16) dft16<true>(&x[b * 16]);
      else if constexpr (R2 == 8) dft8<true>(&x[b * 8]);
      else if constexpr (R2 == 4) dft4<true>(x[b * 4], x[b * 4 + 1], x[b * 4 + 2], x[b * 4 + 3]);
      else dft2(x[b * 2], x[b * 2 + 1]);
    }
    __syncwarp();
#pragma unroll
    for (int b = 0; b < R1 / R2; ++b) {
#pragma unroll
      for (int r = 0; r < R2; ++r) {
        const int s = b * R2 + r;
        *HND_S(&buf[padx<PD>((g + G * b) * R2 + r)]) = make_float4(x[s].re.x, x[s].re.y, x[s].im.x, x[s].im.y);
      }
    }
    __syncwarp();
    float2 u[4];
    load_bases<N>(t, g, u);
    sfor<0, R1>([&](auto rc) {
      constexpr int r = decltype(rc)::value;
      const float4 v = *HND_S(&buf[padx<PD>(g + r * G)]);
      cp y = {make_float2(v.x, v.y), make_float2(v.z, v.w)};
      if constexpr (r > 0) y = ctw<true>(y, w4of(upow<r>(u)));     // W_N^{g r}
      x[r] = y;
    });
    if constexpr (R1 == 16) dft16<true>(x);
    else dft8<true>(x);
  }
}

// Forward padded transform: on entry z[s] = input at natural index g + s G
// (a complex value, the same for both paths); on exit x[s] holds
// (Z[2f], Z[2f+1]) with f = spec_idx<N>(g, s).
template <int N>
__device__ __forceinline__ void padded_fwd(const float2 (&z)[P2<N>::R1], cp (&x)[P2<N>::R1], int g, float4* buf,
                                           int key, Tabs<N> t, unsigned mask) {
  constexpr int G = P2<N>::G, R1 = P2<N>::R1;
  const float2 tg = *HND_S(&t.b[4 * G + g]);
  sfor<0, R1>([&](auto sc) {
    constexpr int s = decltype(sc)::value;
    const float2 w = mul_w32<s * (16 / R1)>(tg);     // W_2N^{g + s G} = W_2N^g W_{2 R1}^s
    const float ore = fmaf(z[s].x, w.x, -z[s].y * w.y);
    const float oim = fmaf(z[s].x, w.y, z[s].y * w.x);
    x[s] = {make_float2(z[s].x, ore), make_float2(z[s].y, oim)};
  });
  fft_fwd<N>(x, g, buf, key, t, mask);
}

// Full (unpadded) forward transform of length 2N: on entry lo[s] = x[g + s G]
// and hi[s] = x[N + g + s G]; on exit x[s] holds (X[2f], X[2f+1]) with
// f = spec_idx<N>(g, s).  Even frequencies are FFT_N(lo + hi), odd ones
// FFT_N((lo - hi) W_2N^j): the two paths of the packed core.
template <int N>
__device__ __forceinline__ void full_fwd(const float2 (&lo)[P2<N>::R1], const float2 (&hi)[P2<N>::R1],
                                         cp (&x)[P2<N>::R1], int g, float4* buf, int key, Tabs<N> t,
                                         unsigned mask) {
  constexpr int G = P2<N>::G, R1 = P2<N>::R1;
  const float2 tg = *HND_S(&t.b[4 * G + g]);
  sfor<0, R1>([&](auto sc) {
    constexpr int s = decltype(sc)::value;
    const float2 w = mul_w32<s * (16 / R1)>(tg);     // W_2N^{g + s G}
    const float2 a = make_float2(lo[s].x + hi[s].x, lo[s].y + hi[s].y);
    const float2 d = make_float2(lo[s].x - hi[s].x, lo[s].y - hi[s].y);
    const float2 b = cmul1(d, w);
    x[s] = {make_float2(a.x, b.x), make_float2(a.y, b.y)};
  });
  fft_fwd<N>(x, g, buf, key, t, mask);
}

// Inverse padded transform keeping outputs [0, N): on entry x[s] =
// (Y[2f], Y[2f+1]); on exit out[s] = y[g + s G] (unnormalised).
template <int N>
__device__ __forceinline__ void padded_inv(cp (&x)[P2<N>::R1], float2 (&out)[P2<N>::R1], int g, float4* buf, int key,
                                           Tabs<N> t, unsigned mask) {
  constexpr int G = P2<N>::G, R1 = P2<N>::R1;
  fft_inv<N>(x, g, buf, key, t, mask);
  const float2 tg = *HND_S(&t.b[4 * G + g]);
  sfor<0, R1>([&](auto sc) {
    constexpr int s = decltype(sc)::value;
    const float2 w = mul_w32<s * (16 / R1)>(tg);   // untwist by conj(W_2N^{g + s G})
    const float re = fmaf(x[s].re.y, w.x, fmaf(x[s].im.y, w.y, x[s].re.x));
    const float im = fmaf(x[s].im.y, w.x, fmaf(-x[s].re.y, w.y, x[s].im.x));
    out[s] = make_float2(re, im);
  });
}

// Partner frequency -k (mod 2N) of spectral slot (f, path): path 0 -> (N - f)
// mod N, path 1 -> N - 1 - f (both as natural half-frequency indices).
template <int N>
__device__ __forceinline__ void fetch_partner(const cp (&x)[P2<N>::R1], cp (&xp)[P2<N>::R1], int g, float4* buf,
                                              int key, unsigned mask) {
  __syncwarp();
#pragma unroll
  for (int s = 0; s < P2<N>::R1; ++s)
    *HND_S(&buf[swz(spec_idx<N>(g, s)) ^ key]) = make_float4(x[s].re.x, x[s].re.y, x[s].im.x, x[s].im.y);
  __syncwarp();
#pragma unroll
  for (int s = 0; s < P2<N>::R1; ++s) {
    const int f = spec_idx<N>(g, s);
    const float4 a = *HND_S(&buf[swz((N - f) & (N - 1)) ^ key]);
    const float4 b = *HND_S(&buf[swz(N - 1 - f) ^ key]);
    xp[s] = {make_float2(a.x, b.y), make_float2(a.z, b.w)};
  }
}

// Row-pair packing: X_a = (Z[k] + conj Z[-k]) / 2, X_b = (Z[k] - conj Z[-k]) / (2i)
__device__ __forceinline__ float2 unpack_a(float2 z, float2 zm) {
  return make_float2(0.5f * (z.x + zm.x), 0.5f * (z.y - zm.y));
}
__device__ __forceinline__ float2 unpack_b(float2 z, float2 zm) {
  return make_float2(0.5f * (z.y + zm.y), 0.5f * (zm.x - z.x));
}
// W[k] = Y_a + i Y_b ; W[-k] = conj(Y_a) + i conj(Y_b)
__device__ __forceinline__ float2 pack_pos(float2 ya, float2 yb) { return make_float2(ya.x - yb.y, ya.y + yb.x); }
__device__ __forceinline__ float2 pack_neg(float2 ya, float2 yb) { return make_float2(ya.x + yb.y, yb.x - ya.y); }

}  // namespace hnd2
