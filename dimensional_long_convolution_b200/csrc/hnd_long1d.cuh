// hnd_long1d.cuh -- 1D grids longer than one transform pencil (n in
// [512, 2^26]): the zero-padded length-P transform (P = 2n) as a multi-level
// split P = P0 P1 (P2) with every factor at most 512, on the row-major view
// [P0][P1][P2] of each grid (j = (j0 P1 + j1) P2 + j2):
//   forward   transform along axis 0 (the padded half j0 >= P0/2 is zero),
//             twiddle W_P^{k0 r} (r the flattened later index), then the same
//             split recursively on the later axes
//             -> X(k0 + P0 k1 + P0 P1 k2) at [k0][k1][k2]
//   modulate  on the last axis (the center)
//   inverse   the same steps in reverse order (last axis first, each twiddle
//             after the transform of its level's later axes): every step is
//             a symmetric operator, so the reversed chain applied to data in
//             split order is the DFT in natural order; on conjugated data it
//             gives the conjugate of the unnormalised inverse at i = j
//   output    y[i] = q[i] (.) for i < n (the crop), optional second gate
// Channel pairs: the inputs of channels 2j and 2j + 1 of one sample are real,
// so they share one complex grid, z = u_a + i u_b.  With Z = U_a + i U_b and
// Z_m = Z(-k), the product that the two channels need is
//   Y = K_a U_a + i K_b U_b = A Z + D conj(Z_m),  A = (K_a + K_b)/2, D = (K_a - K_b)/2
// and the inverse of Y is y_a + i y_b (both convolutions are real).  The
// spectrum of a pair therefore holds (A, D) per frequency, and only for half
// of them: A(-k) = conj A(k), D(-k) = conj D(k).
// (HyenaND pages: arXiv 2607.19378 summary, d = 1 long context through the
// zero-padded FFT path; blog "Native multi-dimensional subquadratic operators
// via input-dependent long convolutions", section "HyenaND".)
// The filter's axis transforms are k_fft_axis2 of hnd_filter2.cuh.
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

// Pair spectrum layout.  The center axis is the last level (length Pc); the
// earlier levels form the pencil frequency kap = k0 + P0 k1 in [0, Po)
// (Po = P / Pc), so k = kap + Po kc.  The pencil of -k is Po - kap (mod Po)
// with kc reversed (Pc - 1 - kc) for kap != 0, and kc negated for kap = 0.
// Pencils kap = 0 and kap = Po/2 are their own partners; the others pair up.
// The spectrum of channel pair j keeps the pencils kap = 0 .. Po/2 only:
//   float4 {A, D} at [j][kap][kc],  (Po/2 + 1) Pc per pair.
// Memory pencil (row-major grid) of pencil frequency kap.
__host__ __device__ __forceinline__ long long l1_pencil(long long kap, int P0, int Pm) {
  return (kap % P0) * Pm + kap / P0;
}
// Grid position of frequency k (split order).
__host__ __device__ __forceinline__ long long l1_pos(long long k, int P0, int Pm, int Pc) {
  const long long Po = static_cast<long long>(P0) * Pm;
  return l1_pencil(k % Po, P0, Pm) * Pc + k / Po;
}

struct L1Spec {
  int P0, Pm, Pc;            // first, middle (1 for two levels) and center factors
  long long Po, R;           // pencils per grid, stored pencils per pair (Po/2 + 1)
  __host__ __device__ long long per_pair() const { return R * Pc; }      // float4
};

// the pair layout of an m-level split P[0..m-1]
inline L1Spec l1_spec_of(int m, const int* P) {
  L1Spec d;
  d.P0 = P[0];
  d.Pm = m == 3 ? P[1] : 1;
  d.Pc = P[m - 1];
  d.Po = static_cast<long long>(d.P0) * d.Pm;
  d.R = d.Po / 2 + 1;
  return d;
}

// filter grids (channels c0 + 2jp + {0, 1} as the real and imaginary part,
// after the forward split transform) -> pair spectrum, scaled by 1/P
static __global__ void k_l1_pair_store(const float2* __restrict__ grid, float4* __restrict__ spec, L1Spec d, int jp0,
                                       int ngrids, float scale) {
  const long long P = d.Po * d.Pc, per = d.per_pair();
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < per * ngrids;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long jp = e / per, rem = e % per, kap = rem / d.Pc, kc = rem % d.Pc;
    const long long k = kap + d.Po * kc, km = (P - k) % P;
    const float2* gj = grid + jp * P;
    const float2 w = *HND_G(&gj[l1_pos(k, d.P0, d.Pm, d.Pc)]);
    const float2 wm = *HND_G(&gj[l1_pos(km, d.P0, d.Pm, d.Pc)]);
    // K_a = (W + conj Wm)/2, K_b = (W - conj Wm)/(2i)
    const float2 ka = make_float2(0.5f * (w.x + wm.x), 0.5f * (w.y - wm.y));
    const float2 kb = make_float2(0.5f * (w.y + wm.y), 0.5f * (wm.x - w.x));
    const float h = 0.5f * scale;
    *HND_G(&spec[(jp0 + jp) * per + rem]) =
        make_float4(h * (ka.x + kb.x), h * (ka.y + kb.y), h * (ka.x - kb.x), h * (ka.y - kb.y));
  }
}

// (A, D) of frequency k from the stored half, conjugated for the other half
__device__ __forceinline__ float4 l1_pair_at(const float4* __restrict__ sp, const L1Spec& d, long long k) {
  const long long kap = k % d.Po, kc = k / d.Po;
  if (kap <= d.Po / 2) return *HND_G(&sp[kap * d.Pc + kc]);
  const float4 v = *HND_G(&sp[(d.Po - kap) * d.Pc + (d.Pc - 1 - kc)]);
  return make_float4(v.x, -v.y, v.z, -v.w);
}

// pair spectra [ceil(C/2)] <-> natural half spectra [C][n + 1]
static __global__ void k_l1_spec_export(const float4* __restrict__ lib, float2* __restrict__ nat, int n, L1Spec d,
                                        long long C) {
  const long long H = n + 1LL;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < H * C;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long c = e / H, k = e % H;
    const float4 ad = l1_pair_at(lib + (c / 2) * d.per_pair(), d, k);
    // K_a = A + D, K_b = A - D
    *HND_G(&nat[e]) = (c & 1) ? make_float2(ad.x - ad.z, ad.y - ad.w) : make_float2(ad.x + ad.z, ad.y + ad.w);
  }
}

__device__ __forceinline__ float2 l1_nat_at(const float2* __restrict__ nat, long long P, int n, long long k) {
  if (k <= n) return *HND_G(&nat[k]);
  const float2 s = *HND_G(&nat[P - k]);
  return make_float2(s.x, -s.y);
}

static __global__ void k_l1_spec_import(const float2* __restrict__ nat, float4* __restrict__ lib, int n, L1Spec d,
                                        long long C, long long pitch) {
  const long long P = d.Po * d.Pc, per = d.per_pair(), npair = (C + 1) / 2;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < per * npair;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long j = e / per, rem = e % per;
    const long long k = rem / d.Pc + d.Po * (rem % d.Pc);
    const float2 ka = l1_nat_at(nat + 2 * j * pitch, P, n, k);
    const float2 kb = 2 * j + 1 < C ? l1_nat_at(nat + (2 * j + 1) * pitch, P, n, k) : make_float2(0.f, 0.f);
    *HND_G(&lib[e]) = make_float4(0.5f * (ka.x + kb.x), 0.5f * (ka.y + kb.y), 0.5f * (ka.x - kb.x),
                                  0.5f * (ka.y - kb.y));
  }
}

// ------------------------------------------------------------ fused passes
// One convolution over a wave of channel pairs as 2m - 1 passes, each an axis
// transform with its neighbours' elementwise steps folded in:
//   kFirst   axis 0: k v of both channels of the pair (real and imaginary
//            part) on the first P0/2 rows (the rest is the zero pad), padded
//            forward transform, forward twiddle of level 0
//   kFwdMid  axis 1 of 3: full forward transform, forward twiddle of level 1
//   center   last axis (k_l1_center): the pencils kap and Po - kap together,
//            full forward transforms, Y = A Z + D conj(Z_m), full inverse
//            transforms, conjugate twiddle of level m - 2
//   kInvMid  axis 1 of 3: full inverse transform, conjugate twiddle of level 0
//   kLast    axis 0: inverse transform of which only the first P0/2 outputs
//            (the crop i < n) are formed; real part to channel a, imaginary
//            part to channel b, output gate(s)
// The inverse chain (inverse transforms, conjugate twiddles, last axis first)
// is the adjoint of the forward chain, so on spectra in split order it forms
// the unnormalised inverse in natural order (the spectrum holds the 1/P).
enum L1Kind { kFirst = 0, kFwdMid = 1, kInvMid = 3, kLast = 4 };

struct L1PassArgs {
  float2* grid;              // wave grids [pair][P]
  long long P;               // points per grid
  long long stride;          // stride of the pass's axis (points)
  long long npen;            // pencils in the wave (center: pencil pairs)
  long long twQ;             // twiddle order Q (W_Q)
  int twP;                   // inverse twiddles: the level's factor (k = outer index mod twP)
  int lgS, lgP, lgQ;         // log2 of stride, P and twQ (all powers of two)
  int n;                     // volume length
  long long v0;              // first channel pair of the wave (order b H + j)
  int H;                     // channel pairs per sample, (C + 1) / 2
  const void* a;             // kFirst: k
  const void* b;             // kFirst: v
  const void* q;             // kLast: output gate
  void* y;                   // kLast: output
  const void* g2;            // kLast: second gate (dual output) or null
  void* y2;
  const float4* spec;        // center: pair spectra [H] per sample set
  long long sbs4;            // sample-set stride (float4)
  L1Spec sd;                 // center: split of the pair spectrum
  int lgP0;                  // center: log2 P0 (pencil frequency -> memory pencil)
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

// channels of pair pg: first volume (memory order b C + c) and whether the
// second channel exists (odd C leaves the last pair of a sample half empty)
__device__ __forceinline__ long long l1_pair_vol(long long pg, int H, int C, bool* has_b) {
  const long long b = pg / H, j = pg - b * H;
  *has_b = 2 * j + 1 < C;
  return b * C + 2 * j;
}

template <int N, int KIND, class T, bool DUAL>
__global__ void __launch_bounds__(kAT, 2) k_l1_pass(const L1PassArgs a) {
  constexpr int G = P2<N>::G, R1 = P2<N>::R1, PPW = 32 / G, P = 2 * N;
  extern __shared__ __align__(16) unsigned char asmem[];
  pdl_release();
  const Tabs<N> t = tabs_at<N>(asmem);
  float4* xb = reinterpret_cast<float4*>(asmem + Tabs<N>::kBytes);
  tabs_build<N>(t, g_tw512);
  __syncthreads();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pen = lane / G, g = lane % G;
  float4* buf = xb + warp * XB<N>::kWarp + pen * XB<N>::kPen;
  const long long per_cta = (kAT / 32) * PPW;
  const long long S = a.stride;
  const float invQ = ldexpf(1.f, -a.lgQ);
  // twiddle exponents are taken mod Q (Q <= 2^27 a power of two, so 32-bit
  // unsigned products that wrap keep their value mod Q)
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
      bool has_b;
      const long long row0 = l1_pair_vol(a.v0 + vol, a.H, a.C, &has_b) * a.n + i;
      const bool actb = act && has_b;
#pragma unroll
      for (int s = 0; s < R1; ++s) {
        const long long j = row0 + static_cast<long long>(g + s * G) * S;
        z[s] = make_float2(act ? Act<T>::ld_g(ka + j) * Act<T>::ld_g(va + j) : 0.f,
                           actb ? Act<T>::ld_g(ka + j + a.n) * Act<T>::ld_g(va + j + a.n) : 0.f);
      }
      padded_fwd<N>(z, x, g, buf, 0, t, 0u);
    } else if constexpr (KIND == kFwdMid) {
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
    // kLast: with 8 slots a lane, the output gates are loaded before the
    // inverse transform, so that their latency overlaps it (the pass is
    // otherwise bound by waiting on these strided loads); with 16 slots the
    // registers are not there, and they are loaded at the store
    constexpr bool PRE = KIND == kLast && R1 == 8;
    constexpr int RQ = PRE ? R1 : 1;
    float qa_v[RQ], qb_v[RQ], ga_v[PRE && DUAL ? RQ : 1], gb_v[PRE && DUAL ? RQ : 1];
    bool has_b = false;
    long long orow = 0;
    if constexpr (KIND == kLast) orow = l1_pair_vol(a.v0 + vol, a.H, a.C, &has_b) * a.n + i;
    if constexpr (PRE) {
      const T* qa = static_cast<const T*>(a.q);
#pragma unroll
      for (int s = 0; s < R1; ++s) {
        const long long j = orow + static_cast<long long>(g + s * G) * S;
        qa_v[s] = act ? Act<T>::ld_g(qa + j) : 0.f;
        qb_v[s] = act && has_b ? Act<T>::ld_g(qa + j + a.n) : 0.f;
        if constexpr (DUAL) {
          const T* g2 = static_cast<const T*>(a.g2);
          ga_v[s] = act ? Act<T>::ld_g(g2 + j) : 0.f;
          gb_v[s] = act && has_b ? Act<T>::ld_g(g2 + j + a.n) : 0.f;
        }
      }
    }

    if constexpr (KIND == kFirst || KIND == kFwdMid) {
      // forward twiddle W_Q^{k i} at k = 2f, 2f + 1; store in spectral
      // positions.  With 2f i = 2i (g + G (s / R2) + R1 (s % R2)) the lane
      // builds its twiddles from four exact ones by products (a few float
      // roundings each) instead of one sine-cosine per slot.
      const unsigned qm = (1u << a.lgQ) - 1u;
      const float2 wi = l1_w(i & qm, invQ);
      const float2 bG = l1_w((2u * G * i) & qm, invQ);
      const float2 bR = l1_w((2u * R1 * i) & qm, invQ);
      float2 wo = l1_w((2u * g * i) & qm, invQ), w0 = wo;
#pragma unroll
      for (int s = 0; s < R1; ++s) {
        if (s > 0) {
          if (s % P2<N>::R2 == 0) {
            wo = cmul1(wo, bG);
            w0 = wo;
          } else {
            w0 = cmul1(w0, bR);
          }
        }
        const unsigned f = spec_idx<N>(g, s);
        const float2 w1 = cmul1(w0, wi);
        if (act) {
          *HND_G(&base[(2 * f) * S]) = cmul1(make_float2(x[s].re.x, x[s].im.x), w0);
          *HND_G(&base[(2 * f + 1) * S]) = cmul1(make_float2(x[s].re.y, x[s].im.y), w1);
        }
      }
    } else if constexpr (KIND == kInvMid) {
      float2 lo[R1], hi[R1];
      l1_full_inv<N>(x, lo, hi, g, buf, t);
      // conjugate twiddle of level 0: conj W_P^{k0 (e S + i)}, k0 = o mod twP
      // (exponents mod Q, Q a power of two dividing 2^32; w0 for slot s is
      // conj W^{k (g S + i)} conj W^{k G S}^s)
      const unsigned k = static_cast<unsigned>(o & (a.twP - 1));
      const unsigned Su = static_cast<unsigned>(S);
      const unsigned qm = (1u << a.lgQ) - 1u;
      const float2 wk = l1_conj(l1_w((k * N * Su) & qm, invQ));
      const float2 cG = l1_conj(l1_w((k * G * Su) & qm, invQ));
      float2 w0 = l1_conj(l1_w((k * (static_cast<unsigned>(g) * Su + i)) & qm, invQ));
#pragma unroll
      for (int s = 0; s < R1; ++s) {
        const long long j = g + s * G;
        if (s > 0) w0 = cmul1(w0, cG);
        const float2 w1 = cmul1(w0, wk);
        if (act) {
          *HND_G(&base[j * S]) = cmul1(lo[s], w0);
          *HND_G(&base[(j + N) * S]) = cmul1(hi[s], w1);
        }
      }
    } else {
      // kLast: outputs i0 < N only (the crop); real part -> channel a,
      // imaginary part -> channel b; output gate(s)
      float2 out[R1];
      padded_inv<N>(x, out, g, buf, 0, t, 0u);
      T* ya = static_cast<T*>(a.y);
      const T* qa = static_cast<const T*>(a.q);
      const T* g2 = static_cast<const T*>(a.g2);
#pragma unroll
      for (int s = 0; s < R1; ++s) {
        const long long j = orow + static_cast<long long>(g + s * G) * S;
        if (act) {
          Act<T>::st_g(ya + j, out[s].x * (PRE ? qa_v[s % RQ] : Act<T>::ld_g(qa + j)));
          if constexpr (DUAL)
            Act<T>::st_g(static_cast<T*>(a.y2) + j, out[s].x * (PRE ? ga_v[s % RQ] : Act<T>::ld_g(g2 + j)));
          if (has_b) {
            Act<T>::st_g(ya + j + a.n, out[s].y * (PRE ? qb_v[s % RQ] : Act<T>::ld_g(qa + j + a.n)));
            if constexpr (DUAL)
              Act<T>::st_g(static_cast<T*>(a.y2) + j + a.n,
                           out[s].y * (PRE ? gb_v[s % RQ] : Act<T>::ld_g(g2 + j + a.n)));
          }
        }
      }
    }
  }
}

// Center pass: one unit = the pencil frequencies kap and Po - kap of one
// channel-pair grid, on two neighbouring pencil slots of a warp (side 0 and
// side 1); the self-paired pencils kap = 0 and kap = Po/2 use side 0 alone.
// After the forward transforms each pencil leaves its spectrum in its own
// exchange buffer, and each side reads its partner's values Z_m there:
//   side 0 (kap):       Y[kc] = A[kc] Z[kc] + D[kc] conj(Z_m[pi(kc)])
//   side 1 (Po - kap):  Y[j]  = conj(A[pi(j)]) Z[j] + conj(D[pi(j)]) conj(Z_m[pi(j)])
// with pi(kc) = Pc - 1 - kc (kap != 0) or -kc mod Pc (kap = 0), and (A, D)
// of the stored pencil kap; the adjoint conjugates (A, D) once more.
template <int N>
__global__ void __launch_bounds__(kAT, 2) k_l1_center(const L1PassArgs a) {
  constexpr int G = P2<N>::G, R1 = P2<N>::R1, PPW = 32 / G, UPW = PPW / 2, Pc = 2 * N;
  static_assert(PPW >= 2, "a unit takes two pencil slots of one warp");
  extern __shared__ __align__(16) unsigned char asmem[];
  pdl_release();
  const Tabs<N> t = tabs_at<N>(asmem);
  float4* xb = reinterpret_cast<float4*>(asmem + Tabs<N>::kBytes);
  tabs_build<N>(t, g_tw512);
  __syncthreads();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pen = lane / G, g = lane % G, side = pen & 1;
  float4* buf = xb + warp * XB<N>::kWarp + pen * XB<N>::kPen;
  const float4* pbuf = xb + warp * XB<N>::kWarp + (pen ^ 1) * XB<N>::kPen;
  const L1Spec& d = a.sd;
  const unsigned Po = static_cast<unsigned>(d.Po), R = static_cast<unsigned>(d.R);
  const unsigned total = static_cast<unsigned>(a.npen);            // units in the wave
  const unsigned per_cta = (kAT / 32) * UPW;
  const float invQ = ldexpf(1.f, -a.lgQ);
  const bool conj_spec = a.sconj < 0.f;
  for (unsigned u0 = blockIdx.x * per_cta; u0 < total; u0 += gridDim.x * per_cta) {
    const unsigned u = u0 + warp * UPW + (pen >> 1);
    const bool valid = u < total;
    const unsigned wv = valid ? u / R : 0u, r = valid ? u - wv * R : 0u;
    const bool self = (r == 0u) || (r == Po / 2);
    const bool act = valid && (side == 0 || !self);
    const unsigned kap = side == 0 ? r : (self ? r : Po - r);
    const long long o = (static_cast<long long>(kap & (d.P0 - 1)) * d.Pm) + (kap >> a.lgP0);
    float2* base = a.grid + (static_cast<long long>(wv) * Po + o) * Pc;
    const long long pg = a.v0 + wv;                 // the channel pair
    const long long smp = pg / a.H, jj = pg - smp * a.H;
    const float4* row = a.spec + smp * a.sbs4 + jj * d.per_pair() + static_cast<long long>(r) * Pc;
    // the unit's spectrum row (Pc float4) into L2 while the transforms run
    if (valid && side == 0) {
      for (int q = g; q < Pc / 8; q += G)
        if (HND_RANGE_OK(row + 8 * q, 16)) asm volatile("prefetch.global.L2 [%0];" ::"l"(row + 8 * q));
    }
    float2 lo[R1], hi[R1];
#pragma unroll
    for (int s = 0; s < R1; ++s) {
      const int j = g + s * G;
      lo[s] = act ? *HND_G(&base[j]) : make_float2(0.f, 0.f);
      hi[s] = act ? *HND_G(&base[j + N]) : make_float2(0.f, 0.f);
    }
    cp x[R1];
    full_fwd<N>(lo, hi, x, g, buf, 0, t, 0u);
    // every pencil's spectrum into its exchange buffer, slot f holding
    // (Z[2f], Z[2f + 1])
    __syncwarp();
#pragma unroll
    for (int s = 0; s < R1; ++s)
      *HND_S(&buf[swz(spec_idx<N>(g, s))]) = make_float4(x[s].re.x, x[s].re.y, x[s].im.x, x[s].im.y);
    __syncwarp();
    const float4* src = self ? buf : pbuf;
    const bool flip = (side == 1) != conj_spec;
#pragma unroll
    for (int s = 0; s < R1; ++s) {
      const int f = spec_idx<N>(g, s);
      // partner values at pi(2f) and pi(2f + 1)
      float2 zm0, zm1;
      if (r == 0u && side == 0) {
        const float4 pa = *HND_S(&src[swz((N - f) & (N - 1))]);     // -2f: slot (N - f) mod N, path 0
        const float4 pb = *HND_S(&src[swz(N - 1 - f)]);             // -(2f + 1): slot N - 1 - f, path 1
        zm0 = make_float2(pa.x, pa.z);
        zm1 = make_float2(pb.y, pb.w);
      } else {
        const float4 pb = *HND_S(&src[swz(N - 1 - f)]);             // Pc - 1 - 2f: path 1; Pc - 2 - 2f: path 0
        zm0 = make_float2(pb.y, pb.w);
        zm1 = make_float2(pb.x, pb.z);
      }
      // (A, D) of the stored pencil at kc (side 0) or pi(kc) (side 1)
      float4 s0 = make_float4(0.f, 0.f, 0.f, 0.f), s1 = s0;
      if (act) {
        s0 = __ldg(HND_G(row + (side == 0 ? 2 * f : Pc - 1 - 2 * f)));
        s1 = __ldg(HND_G(row + (side == 0 ? 2 * f + 1 : Pc - 2 - 2 * f)));
      }
      if (flip) {
        s0.y = -s0.y;
        s0.w = -s0.w;
        s1.y = -s1.y;
        s1.w = -s1.w;
      }
      // Y = A Z + D conj(Z_m)
      const float2 z0 = make_float2(x[s].re.x, x[s].im.x), z1 = make_float2(x[s].re.y, x[s].im.y);
      const float y0r = s0.x * z0.x - s0.y * z0.y + s0.z * zm0.x + s0.w * zm0.y;
      const float y0i = s0.x * z0.y + s0.y * z0.x + s0.w * zm0.x - s0.z * zm0.y;
      const float y1r = s1.x * z1.x - s1.y * z1.y + s1.z * zm1.x + s1.w * zm1.y;
      const float y1i = s1.x * z1.y + s1.y * z1.x + s1.w * zm1.x - s1.z * zm1.y;
      x[s] = {make_float2(y0r, y1r), make_float2(y0i, y1i)};
    }
    __syncwarp();                                   // the partner is done with this buffer
    l1_full_inv<N>(x, lo, hi, g, buf, t);
    // conjugate twiddle of the previous level: conj W_Q^{k e}, k = o mod twP,
    // e the element's index along this (last) axis
    // (w0 for slot s is conj W^{k g} conj W^{k G}^s)
    const unsigned k = static_cast<unsigned>(o & (a.twP - 1));
    const unsigned qm = (1u << a.lgQ) - 1u;
    const float2 wk = l1_conj(l1_w((k * N) & qm, invQ));
    const float2 cG = l1_conj(l1_w((k * G) & qm, invQ));
    float2 w0 = l1_conj(l1_w((k * g) & qm, invQ));
#pragma unroll
    for (int s = 0; s < R1; ++s) {
      const unsigned j = g + s * G;
      if (s > 0) w0 = cmul1(w0, cG);
      const float2 w1 = cmul1(w0, wk);
      if (act) {
        *HND_G(&base[j]) = cmul1(lo[s], w0);
        *HND_G(&base[j + N]) = cmul1(hi[s], w1);
      }
    }
  }
}

// The middle axis passes (kFwdMid, kInvMid) for pencils of 8 slots a lane
// (N <= 64), with two pencil groups a CTA iteration: both groups' strided
// loads are issued before the first group's transform, so the second group's
// latency overlaps it (the same arithmetic as k_l1_pass; with 16 slots a
// lane the second group's registers spill, and k_l1_pass runs instead).
template <int N, bool INV>
__global__ void __launch_bounds__(kAT, 2) k_l1_mid2g(const L1PassArgs a) {
  constexpr int G = P2<N>::G, R1 = P2<N>::R1, PPW = 32 / G, P = 2 * N;
  extern __shared__ __align__(16) unsigned char asmem[];
  pdl_release();
  const Tabs<N> t = tabs_at<N>(asmem);
  float4* xb = reinterpret_cast<float4*>(asmem + Tabs<N>::kBytes);
  tabs_build<N>(t, g_tw512);
  __syncthreads();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pen = lane / G, g = lane % G;
  float4* buf = xb + warp * XB<N>::kWarp + pen * XB<N>::kPen;
  const long long per_cta = (kAT / 32) * PPW;
  const long long S = a.stride;
  const float invQ = ldexpf(1.f, -a.lgQ);
  const unsigned qm = (1u << a.lgQ) - 1u;
  for (long long p0 = static_cast<long long>(blockIdx.x) * 2 * per_cta; p0 < a.npen;
       p0 += static_cast<long long>(gridDim.x) * 2 * per_cta) {
    long long pp[2];
    bool act[2];
    long long o[2];
    unsigned ii[2];
    float2* base[2];
    float2 va[2][R1], vb[2][R1];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      pp[h] = p0 + h * per_cta + warp * PPW + pen;
      act[h] = pp[h] < a.npen;
      o[h] = act[h] ? pp[h] >> a.lgS : 0;
      ii[h] = act[h] ? static_cast<unsigned>(pp[h] & (S - 1)) : 0u;
      base[h] = a.grid + (((o[h] * P) << a.lgS) + ii[h]);
#pragma unroll
      for (int s = 0; s < R1; ++s) {
        const long long j = INV ? 2LL * spec_idx<N>(g, s) : static_cast<long long>(g + s * G);
        va[h][s] = act[h] ? *HND_G(&base[h][j * S]) : make_float2(0.f, 0.f);
        vb[h][s] = act[h] ? *HND_G(&base[h][(INV ? j + 1 : j + N) * S]) : make_float2(0.f, 0.f);
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      cp x[R1];
      const unsigned i = ii[h];
      if constexpr (!INV) {
        full_fwd<N>(va[h], vb[h], x, g, buf, 0, t, 0u);
        const float2 wi = l1_w(i & qm, invQ);
        const float2 bG = l1_w((2u * G * i) & qm, invQ);
        const float2 bR = l1_w((2u * R1 * i) & qm, invQ);
        float2 wo = l1_w((2u * g * i) & qm, invQ), w0 = wo;
#pragma unroll
        for (int s = 0; s < R1; ++s) {
          if (s > 0) {
            if (s % P2<N>::R2 == 0) {
              wo = cmul1(wo, bG);
              w0 = wo;
            } else {
              w0 = cmul1(w0, bR);
            }
          }
          const unsigned f = spec_idx<N>(g, s);
          const float2 w1 = cmul1(w0, wi);
          if (act[h]) {
            *HND_G(&base[h][(2 * f) * S]) = cmul1(make_float2(x[s].re.x, x[s].im.x), w0);
            *HND_G(&base[h][(2 * f + 1) * S]) = cmul1(make_float2(x[s].re.y, x[s].im.y), w1);
          }
        }
      } else {
#pragma unroll
        for (int s = 0; s < R1; ++s) x[s] = {make_float2(va[h][s].x, vb[h][s].x), make_float2(va[h][s].y, vb[h][s].y)};
        float2 lo[R1], hi[R1];
        l1_full_inv<N>(x, lo, hi, g, buf, t);
        const unsigned k = static_cast<unsigned>(o[h] & (a.twP - 1));
        const unsigned Su = static_cast<unsigned>(S);
        const float2 wk = l1_conj(l1_w((k * N * Su) & qm, invQ));
        const float2 cG = l1_conj(l1_w((k * G * Su) & qm, invQ));
        float2 w0 = l1_conj(l1_w((k * (static_cast<unsigned>(g) * Su + i)) & qm, invQ));
#pragma unroll
        for (int s = 0; s < R1; ++s) {
          const long long j = g + s * G;
          if (s > 0) w0 = cmul1(w0, cG);
          const float2 w1 = cmul1(w0, wk);
          if (act[h]) {
            *HND_G(&base[h][j * S]) = cmul1(lo[s], w0);
            *HND_G(&base[h][(j + N) * S]) = cmul1(hi[s], w1);
          }
        }
      }
    }
  }
}

}  // namespace hnd2
