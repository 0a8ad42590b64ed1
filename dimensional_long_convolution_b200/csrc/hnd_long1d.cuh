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

#include "hnd_filter2.cuh"

namespace hnd2 {

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
    const float2 x = *HND_G(&grid[e]);
    *HND_G(&grid[e]) = make_float2(x.x * c - x.y * s, x.x * s + x.y * c);
  }
}

// filter grids (after the forward split transform) -> spectrum [c0 + c][P], scaled
static __global__ void k_l1_spec_store(const float2* __restrict__ grid, float2* __restrict__ spec, long long P, int c0,
                                       int nc, float scale) {
  const long long total = P * nc;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float2 x = *HND_G(&grid[e]);
    *HND_G(&spec[static_cast<long long>(c0) * P + e]) = make_float2(x.x * scale, x.y * scale);
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
    *HND_G(&nat[e]) = *HND_G(&lib[c * P + l1_pos(k, P0, P1, P2)]);
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
      s = *HND_G(&nat[c * pitch + k]);
    } else {
      s = *HND_G(&nat[c * pitch + (P - k)]);
      s.y = -s.y;
    }
    *HND_G(&lib[e]) = make_float2(s.x * scale, s.y * scale);
  }
}

// ------------------------------------------------------------ fused passes
// One convolution over a wave of volumes as 2m - 1 passes, each an axis
// transform with its neighbours' elementwise steps folded in:
//   kFirst   axis 0: k v of the first P0/2 rows (the rest is the zero pad),
//            padded forward transform, forward twiddle of level 0
//   kFwdMid  axis 1 of 3: full forward transform, forward twiddle of level 1
//   kCenter  last axis: full forward transform, spectrum product, full
//            inverse transform, conjugate twiddle of level m - 2
//   kInvMid  axis 1 of 3: full inverse transform, conjugate twiddle of level 0
//   kLast    axis 0: inverse transform of which only the first P0/2 outputs
//            (the crop i < n) are formed, output gate(s)
// The inverse chain (inverse transforms, conjugate twiddles, last axis first)
// is the adjoint of the forward chain, so on spectra in split order it forms
// the unnormalised inverse in natural order (the spectrum holds the 1/P).
enum L1Kind { kFirst = 0, kFwdMid = 1, kCenter = 2, kInvMid = 3, kLast = 4 };

struct L1PassArgs {
  float2* grid;              // wave grids [vol][P]
  long long P;               // points per grid
  long long stride;          // stride of the pass's axis (points)
  long long npen;            // pencils in the wave
  long long twQ;             // twiddle order Q (W_Q)
  int twP;                   // inverse twiddles: the level's factor (k = outer index mod twP)
  int lgS, lgP, lgQ;         // log2 of stride, P and twQ (all powers of two)
  int n;                     // volume length
  long long v0;              // first volume of the wave (memory order b C + c)
  const void* a;             // kFirst: k
  const void* b;             // kFirst: v
  const void* q;             // kLast: output gate
  void* y;                   // kLast: output
  const void* g2;            // kLast: second gate (dual output) or null
  void* y2;
  const float2* spec;        // kCenter: spectrum [C][P] per sample set
  long long sbs;             // sample-set stride (complex values)
  float sconj;               // -1: conjugate spectrum (adjoint)
  int C;
};

// W_Q^m for 0 <= m < Q, with invQ = 1/Q exact (Q a power of two): the
// ratio m/Q is exact while m < 2^24
__device__ __forceinline__ float2 l1_w(unsigned m, float invQ) {
  float s, c;
  sincospif(-2.f * (static_cast<float>(m) * invQ), &s, &c);
  return make_float2(c, s);
}

__device__ __forceinline__ float2 l1_conj(float2 a) { return make_float2(a.x, -a.y); }

template <int N>
__device__ __forceinline__ void l1_full_inv(cp (&x)[P2<N>::R1], float2 (&lo)[P2<N>::R1], float2 (&hi)[P2<N>::R1],
                                            int g, float4* buf, Tabs<N> t) {
  constexpr int G = P2<N>::G, R1 = P2<N>::R1;
  fft_inv<N>(x, g, buf, 0, t, 0u);
  const float2 tg = *HND_S(&t.b[4 * G + g]);
  sfor<0, R1>([&](auto sc) {
    constexpr int s = decltype(sc)::value;
    const float2 w = mul_w32<s * (16 / R1)>(tg);     // W_2N^{g + s G}
    // path 0: A_j, path 1: B_j; y[j] = A + B conj(w), y[j + N] = A - B conj(w)
    const float br = fmaf(x[s].re.y, w.x, x[s].im.y * w.y);
    const float bi = fmaf(x[s].im.y, w.x, -x[s].re.y * w.y);
    lo[s] = make_float2(x[s].re.x + br, x[s].im.x + bi);
    hi[s] = make_float2(x[s].re.x - br, x[s].im.x - bi);
  });
}

template <int N, int KIND, class T, bool DUAL>
__global__ void __launch_bounds__(kAT, 2) k_l1_pass(const L1PassArgs a) {
  constexpr int G = P2<N>::G, R1 = P2<N>::R1, PPW = 32 / G, P = 2 * N;
  extern __shared__ __align__(16) unsigned char asmem[];
  const Tabs<N> t = tabs_at<N>(asmem);
  float4* xb = reinterpret_cast<float4*>(asmem + Tabs<N>::kBytes);
  tabs_build<N>(t, g_tw512);
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pen = lane / G, g = lane % G;
  float4* buf = xb + warp * XB<N>::kWarp + pen * XB<N>::kPen;
  const long long per_cta = (kAT / 32) * PPW;
  const long long S = a.stride;
  const float invQ = ldexpf(1.f, -a.lgQ);
  // every product below is < Q <= 2^27 (the level's factor times the index
  // range of the later levels), so 32-bit unsigned arithmetic is exact
  for (long long p0 = static_cast<long long>(blockIdx.x) * per_cta; p0 < a.npen;
       p0 += static_cast<long long>(gridDim.x) * per_cta) {
    const long long p = p0 + warp * PPW + pen;
    const bool act = p < a.npen;
    const long long o = act ? p >> a.lgS : 0;
    const unsigned i = act ? static_cast<unsigned>(p & (S - 1)) : 0u;
    const long long start = ((o * P) << a.lgS) + i;   // first point of the pencil in the wave
    const long long vol = start >> a.lgP;             // the pencil's volume within the wave
    float2* base = a.grid + start;
    cp x[R1];
    if constexpr (KIND == kFirst) {
      const T* ka = static_cast<const T*>(a.a);
      const T* va = static_cast<const T*>(a.b);
      float2 z[R1];
      const long long row0 = (a.v0 + vol) * a.n + i;
#pragma unroll
      for (int s = 0; s < R1; ++s) {
        const long long j = row0 + static_cast<long long>(g + s * G) * S;
        z[s] = act ? make_float2(Act<T>::ld_g(ka + j) * Act<T>::ld_g(va + j), 0.f) : make_float2(0.f, 0.f);
      }
      padded_fwd<N>(z, x, g, buf, 0, t, 0u);
    } else if constexpr (KIND == kFwdMid || KIND == kCenter) {
      float2 lo[R1], hi[R1];
#pragma unroll
      for (int s = 0; s < R1; ++s) {
        const long long j = g + s * G;
        lo[s] = act ? *HND_G(&base[j * S]) : make_float2(0.f, 0.f);
        hi[s] = act ? *HND_G(&base[(j + N) * S]) : make_float2(0.f, 0.f);
      }
      full_fwd<N>(lo, hi, x, g, buf, 0, t, 0u);
    } else {
      // kInvMid, kLast: spectral input, (Y[2f], Y[2f+1]) per slot
#pragma unroll
      for (int s = 0; s < R1; ++s) {
        const long long f = spec_idx<N>(g, s);
        const float2 e0 = act ? *HND_G(&base[(2 * f) * S]) : make_float2(0.f, 0.f);
        const float2 e1 = act ? *HND_G(&base[(2 * f + 1) * S]) : make_float2(0.f, 0.f);
        x[s] = {make_float2(e0.x, e1.x), make_float2(e0.y, e1.y)};
      }
    }

    if constexpr (KIND == kFirst || KIND == kFwdMid) {
      // forward twiddle W_Q^{k i} at k = 2f, 2f + 1; store in spectral positions
      const float2 wi = l1_w(i, invQ);
#pragma unroll
      for (int s = 0; s < R1; ++s) {
        const unsigned f = spec_idx<N>(g, s);
        const float2 w0 = l1_w((2u * f) * i, invQ);
        const float2 w1 = cmul1(w0, wi);
        if (act) {
          *HND_G(&base[(2 * f) * S]) = cmul1(make_float2(x[s].re.x, x[s].im.x), w0);
          *HND_G(&base[(2 * f + 1) * S]) = cmul1(make_float2(x[s].re.y, x[s].im.y), w1);
        }
      }
    } else if constexpr (KIND == kCenter) {
      const int vg = static_cast<int>(a.v0 + vol);     // B C <= INT_MAX
      const long long bb = vg / a.C, cc = vg % a.C;
      const float2* Sp = a.spec + bb * a.sbs + cc * a.P + (start - vol * a.P);
#pragma unroll
      for (int s = 0; s < R1; ++s) {
        const long long f = spec_idx<N>(g, s);
        float4 sv = act ? __ldg(HND_G(reinterpret_cast<const float4*>(Sp + 2 * f))) : make_float4(0.f, 0.f, 0.f, 0.f);
        sv.y *= a.sconj;
        sv.w *= a.sconj;
        const float2 y0 = cmul1(make_float2(x[s].re.x, x[s].im.x), make_float2(sv.x, sv.y));
        const float2 y1 = cmul1(make_float2(x[s].re.y, x[s].im.y), make_float2(sv.z, sv.w));
        x[s] = {make_float2(y0.x, y1.x), make_float2(y0.y, y1.y)};
      }
      float2 lo[R1], hi[R1];
      l1_full_inv<N>(x, lo, hi, g, buf, t);
      // conjugate twiddle of the previous level: conj W_Q^{k e}, k = o mod twP,
      // e the element's index along this (last) axis
      const unsigned k = static_cast<unsigned>(o & (a.twP - 1));
      const float2 wk = l1_conj(l1_w(k * N, invQ));
#pragma unroll
      for (int s = 0; s < R1; ++s) {
        const unsigned j = g + s * G;
        const float2 w0 = l1_conj(l1_w(k * j, invQ));
        const float2 w1 = cmul1(w0, wk);
        if (act) {
          *HND_G(&base[j]) = cmul1(lo[s], w0);
          *HND_G(&base[j + N]) = cmul1(hi[s], w1);
        }
      }
    } else if constexpr (KIND == kInvMid) {
      float2 lo[R1], hi[R1];
      l1_full_inv<N>(x, lo, hi, g, buf, t);
      // conjugate twiddle of level 0: conj W_P^{k0 (e S + i)}, k0 = o mod twP
      const unsigned k = static_cast<unsigned>(o & (a.twP - 1));
      const unsigned Su = static_cast<unsigned>(S);
      const float2 wk = l1_conj(l1_w(k * N * Su, invQ));
#pragma unroll
      for (int s = 0; s < R1; ++s) {
        const long long j = g + s * G;
        const float2 w0 = l1_conj(l1_w(k * (static_cast<unsigned>(j) * Su + i), invQ));
        const float2 w1 = cmul1(w0, wk);
        if (act) {
          *HND_G(&base[j * S]) = cmul1(lo[s], w0);
          *HND_G(&base[(j + N) * S]) = cmul1(hi[s], w1);
        }
      }
    } else {
      // kLast: outputs i0 < N only (the crop), real part, output gate(s)
      float2 out[R1];
      padded_inv<N>(x, out, g, buf, 0, t, 0u);
      const T* qa = static_cast<const T*>(a.q);
      T* ya = static_cast<T*>(a.y);
      const long long row0 = (a.v0 + vol) * a.n + i;
#pragma unroll
      for (int s = 0; s < R1; ++s) {
        const long long j = row0 + static_cast<long long>(g + s * G) * S;
        if (act) {
          Act<T>::st_g(ya + j, out[s].x * Act<T>::ld_g(qa + j));
          if constexpr (DUAL)
            Act<T>::st_g(static_cast<T*>(a.y2) + j, out[s].x * Act<T>::ld_g(static_cast<const T*>(a.g2) + j));
        }
      }
    }
  }
}

}  // namespace hnd2
