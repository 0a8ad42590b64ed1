// hnd_filter2.cuh -- the implicit filter on the offset grid (call 1) as tiled
// fp32 products: per CTA, 128 offsets; their Fourier features and hidden
// layer are computed once into shared memory, then the output layer runs as a
// register-tiled product over tiles of 32 channels of the chunk.
// (HyenaND pages: gist.science summary of arXiv 2607.19378, "Methodologie",
// kernel parameterisation -- a coordinate MLP with sine activation on
// continuous offsets, times a window; blog "Native multi-dimensional
// subquadratic operators via input-dependent long convolutions", section on
// the neural parameterisation.)
//   phi(t) = [sin(pi m t_a / n_a), cos(pi m t_a / n_a)]  m = 1..M, axis-major
//   h = sin(W1 phi + b1),  K_c(t) = (W2 h + b2)_c w_c(t)
//   w_c(t) = exp(-alpha_c |t|_2 / s), or the Gaussian exp(-alpha_c (|t|_2 / s)^2)
// written wrap-placed (offset t at slot t mod P on each axis) into a complex
// grid [nc][P^d] whose other slots the caller has zeroed.
#pragma once

#include <cuda_runtime.h>

#include "hnd_fused2.cuh"     // packed FFT core and the W_512 table

namespace hnd2 {

constexpr int kFT = 256;     // threads per CTA
constexpr int kFO = 128;     // offsets per CTA
constexpr int kFC = 32;      // channels per output tile
constexpr int kFNarrow = 8;  // a tile with at most this many channels left takes the narrow path

struct FilterMlpArgs {
  const float *W1, *b1, *W2, *b2, *alpha;
  int num_freqs, hidden, fin;    // fin = 2 num_freqs ndim
  float decay_scale;
  int window;                    // 0: exp(-alpha |t| / s), 1: exp(-alpha (|t| / s)^2)
  int circular;                  // 1: evaluate at each offset's periodic representative
  int ndim;
  int n[3];
  int c0, nc;                    // channel chunk [c0, c0 + nc)
  float2* grid;                  // [nc][P^d], or with pair: [(nc + 1) / 2][P^d], channel c in component c & 1
  int pair = 0;
  const float* gamma = nullptr;  // FiLM: sin(gamma (W1 phi + b1) + beta), [hidden] each; null = plain
  const float* beta = nullptr;
  const float* tab = nullptr;    // per-axis first-layer tables (k_filter_tables)
  int cgroup = 1 << 30;          // channels per CTA row of the grid (blockIdx.y; a multiple of kFC)
};

// The first layer is separable over the axes: the features of axis a depend on
// t_a alone, so W1 phi(t) = sum_a T_a[t_a] with
//   T_a[h][t_a] = sum_m W1[h, f(a,m,sin)] sin(pi m t_a / n_a) + W1[h, f(a,m,cos)] cos(pi m t_a / n_a),
// tabulated once per call for t_a in [-(n_a - 1), n_a - 1] (index t_a + n_a - 1),
// axis a's table at HP * sum_{b<a} (2 n_b - 1), h-major.  The hidden unit of
// offset t is then sin(b1 + T_0[t_0] + T_1[t_1] + T_2[t_2]) (FiLM applied to
// the sum): ndim table reads per unit instead of 2 M ndim products.
// The last axis L = ndim - 1 varies fastest over a tile of offsets, so the
// sum splits into a row part R = b1 + sum_{a<L} T_a (one value per row of the
// tile) and T_L, and with FiLM's gamma and beta
//   sin(gamma (R + T_L) + beta) = sin(A) cos(gamma T_L) + cos(A) sin(gamma T_L),  A = gamma R + beta:
// sin and cos of gamma T_L follow the tables (k_filter_trig, [HP][E_L] each),
// sin A and cos A are computed once per row and unit, and each hidden unit of
// an offset costs two table reads and two products.
inline long long filter_table_floats(int HP, int ndim, const int* n) {
  long long e = 0;
  for (int a = 0; a < ndim; ++a) e += 2LL * n[a] - 1;
  return (e + 2LL * (2LL * n[ndim - 1] - 1)) * HP;
}
// float offset of the sine table of the last axis (the cosine table follows)
inline __host__ __device__ long long filter_trig_offset(int HP, int ndim, const int* n) {
  long long e = 0;
  for (int a = 0; a < ndim; ++a) e += 2LL * n[a] - 1;
  return e * HP;
}

static __global__ void k_filter_tables(const float* __restrict__ W1, int hidden, int HP, int num_freqs, int ndim,
                                       int n0, int n1, int n2, float* __restrict__ tab) {
  const int nn[3] = {n0, n1, n2};
  const int fin = 2 * num_freqs * ndim;
  long long base = 0;
  for (int a = 0; a < ndim; ++a) {
    const int E = 2 * nn[a] - 1;
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < HP * E; e += gridDim.x * blockDim.x) {
      const int h = e / E, j = e % E;
      const int t = j - (nn[a] - 1);
      float acc = 0.f;
      if (h < hidden) {
        for (int m = 1; m <= num_freqs; ++m) {
          float sv, cv;
          sincospif(static_cast<float>(m) * (static_cast<float>(t) / static_cast<float>(nn[a])), &sv, &cv);
          const int f = 2 * (a * num_freqs + m - 1);
          acc = fmaf(__ldg(HND_G(W1 + static_cast<long long>(h) * fin + f)), sv, acc);
          acc = fmaf(__ldg(HND_G(W1 + static_cast<long long>(h) * fin + f + 1)), cv, acc);
        }
      }
      (*HND_G(&tab[base + e])) = acc;
    }
    base += static_cast<long long>(HP) * E;
  }
}

// sin and cos of gamma_h T_L[h][t] for the last axis (gamma = 1 without FiLM),
// by the full-range library sincosf
static __global__ void k_filter_trig(float* __restrict__ tab, int HP, int hidden, int ndim, int n0, int n1, int n2,
                                     const float* __restrict__ gamma) {
  const int nn[3] = {n0, n1, n2};
  const long long off = filter_trig_offset(HP, ndim, nn);
  const int E = 2 * nn[ndim - 1] - 1;
  const float* TL = tab + off - static_cast<long long>(HP) * E;
  float* S = tab + off;
  float* Cc = S + static_cast<long long>(HP) * E;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < HP * E; e += gridDim.x * blockDim.x) {
    const int h = e / E;
    float x = *HND_G(&TL[e]);
    if (gamma && h < hidden) x *= __ldg(HND_G(gamma + h));
    float sv, cv;
    sincosf(x, &sv, &cv);
    *HND_G(&S[e]) = sv;
    *HND_G(&Cc[e]) = cv;
  }
}

// Shared layout (floats), HP = hidden rounded up to a multiple of 32:
//   [phi[fin][kFO] | w1[fin][HP]] | hid[HP][kFO] | w2[HP][kFC] | b1[HP] | rad[kFO] |
//   slot[kFO] (int) | tix[3][kFO] (int) | {sA, cA}[HP][kFR] | rtix[2][kFR] (int);
//   the bracketed part only on the feature path, the braced one only on the
//   table path
constexpr int kFR = 12;      // rows of the last axis a tile of kFO offsets can touch (2 n_L - 1 >= 15)
template <int HP>
struct FilterSmem {
  static size_t bytes(int fin, bool tab) {
    const size_t feat = tab ? 0 : static_cast<size_t>(fin) * (kFO + HP);
    const size_t rows = tab ? 2 * static_cast<size_t>(HP) * kFR : 0;
    return sizeof(float) * (feat + static_cast<size_t>(HP) * kFO + static_cast<size_t>(HP) * kFC + HP + kFO + rows) +
           sizeof(int) * (4 * kFO + 2 * kFR);
  }
};

// sin(x) for the sine layer: Cody-Waite reduction of x to r = x - 2 pi m in
// [-pi, pi] (m = rint(x / 2 pi), 2 pi split into a head exact in fp32 and a
// tail), then the hardware sine approximation __sinf on r, whose absolute
// error on [-pi, pi] is about 2^-21.  The hidden units feed the kernel
// values, whose spectrum is checked against the float64 oracle at 2e-5.
__device__ __forceinline__ float sine_layer(float x) {
  const float m = rintf(x * 0.15915494309189535f);         // 1 / (2 pi)
  float r = fmaf(m, -6.28125f, x);                          // 2 pi head (exact times m for |m| < 2^15)
  r = fmaf(m, -1.9353071795864769e-3f, r);                  // 2 pi - 6.28125
  return __sinf(r);
}

// Kernel values of channels c .. c + 3 (c a multiple of 4; channels at or
// beyond nc carry 0 and are not stored) at grid slot `so`: one real grid per
// channel, or with pair two channels per complex grid (c even in the real
// part, c + 1 in the imaginary part).
__device__ __forceinline__ void store_k4(const FilterMlpArgs& a, int c, long long gsz, int so, const float (&kv)[4]) {
  if (a.pair) {
#pragma unroll
    for (int j = 0; j < 4; j += 2)
      if (c + j < a.nc) *HND_G(&a.grid[static_cast<long long>((c + j) >> 1) * gsz + so]) = make_float2(kv[j], kv[j + 1]);
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (c + j < a.nc) *HND_G(&a.grid[static_cast<long long>(c + j) * gsz + so]) = make_float2(kv[j], 0.f);
  }
}

template <int HP, bool TAB>
__global__ void __launch_bounds__(kFT) k_filter_mlp2(const FilterMlpArgs a) {
  static_assert(HP % 32 == 0 && HP <= 128, "hidden tile");
  constexpr int HG = HP / 8;                 // hidden outputs per thread in the hidden layer
  extern __shared__ __align__(16) float fsm[];
  const int fin = a.fin;
  float* phi = fsm;                          // [fin][kFO] (feature path)
  float* w1 = phi + (TAB ? 0 : fin * kFO);   // [fin][HP]  (feature path)
  float* hid = w1 + (TAB ? 0 : fin * HP);    // [HP][kFO]
  float* w2 = hid + HP * kFO;                // [HP][kFC]
  float* b1 = w2 + HP * kFC;                 // [HP]
  float* rad = b1 + HP;                      // [kFO]
  int* slot = reinterpret_cast<int*>(rad + kFO);
  int* tix = slot + kFO;                     // [3][kFO]: table column per axis (table path)
  float* sA = reinterpret_cast<float*>(tix + 3 * kFO);   // [HP][kFR] (table path)
  float* cA = sA + HP * kFR;
  int* rtix = reinterpret_cast<int*>(cA + HP * kFR);     // [2][kFR]: the row's columns of axes 0, 1
  const int tid = threadIdx.x;
  // axes as scalars (an unused axis has extent 1 and offset 0)
  const int n0 = a.n[0], n1 = a.ndim > 1 ? a.n[1] : 1, n2 = a.ndim > 2 ? a.n[2] : 1;
  const int E0 = 2 * n0 - 1, E1 = 2 * n1 - 1, E2 = 2 * n2 - 1;
  const int P0 = 2 * n0, P1 = a.ndim > 1 ? 2 * n1 : 1, P2 = a.ndim > 2 ? 2 * n2 : 1;
  const long long noff = static_cast<long long>(E0) * E1 * E2;
  const long long gsz = static_cast<long long>(P0) * P1 * P2;
  const long long e0 = static_cast<long long>(blockIdx.x) * kFO;
  // offset t of tile entry o (the last axis fastest; past the end: the last offset)
  auto offset_of = [&](int o, int& t0, int& t1, int& t2) {
    long long r = e0 + o < noff ? e0 + o : noff - 1;
    const int i2 = static_cast<int>(r % E2);
    r /= E2;
    const int i1 = static_cast<int>(r % E1);
    const int i0 = static_cast<int>(r / E1);
    t0 = i0 - (n0 - 1), t1 = i1 - (n1 - 1), t2 = i2 - (n2 - 1);
  };
  // circular mode: the network sees the representative of t mod n in
  // [-n/2, n/2) (the linear offsets t and t - n then carry the same value,
  // which makes the linear convolution on the 2n grid the circular one)
  auto rep = [&](int t, int n) { return a.circular ? ((t + n / 2) % n + n) % n - n / 2 : t; };

  // first layer weights (zero-padded to HP hidden units: sin(0) = 0 and the
  // padded output weights are zero, so the padding contributes nothing)
  if constexpr (!TAB) {
    for (int i = tid; i < fin * HP; i += kFT) {
      const int f = i / HP, h = i % HP;
      (*HND_S(&w1[i])) = h < a.hidden ? __ldg(HND_G(a.W1 + static_cast<long long>(h) * fin + f)) : 0.f;
    }
  }
  for (int h = tid; h < HP; h += kFT) (*HND_S(&b1[h])) = h < a.hidden ? __ldg(HND_G(a.b1 + h)) : 0.f;
  // offsets of this tile: radius and slot (offset t at t mod P per axis)
  for (int o = tid; o < kFO; o += kFT) {
    int t0, t1, t2;
    offset_of(o, t0, t1, t2);
    const float f0 = static_cast<float>(rep(t0, n0)), f1 = static_cast<float>(rep(t1, n1)),
                f2 = static_cast<float>(rep(t2, n2));
    // the window's argument |t| / s, squared for the Gaussian window
    const float rs = sqrtf(f0 * f0 + f1 * f1 + f2 * f2) / a.decay_scale;
    (*HND_S(&rad[o])) = a.window == 1 ? rs * rs : rs;
    const int s0 = (t0 + P0) % P0, s1 = (t1 + P1) % P1, s2 = (t2 + P2) % P2;
    (*HND_S(&slot[o])) = (s0 * P1 + s1) * P2 + s2;
    if constexpr (TAB) {
      // tix[0]: the tile row of the offset; tix[1]: its last-axis column
      const int la = a.ndim - 1;
      const int EL = la == 0 ? E0 : (la == 1 ? E1 : E2);
      const int tl = la == 0 ? t0 : (la == 1 ? t1 : t2), nl = la == 0 ? n0 : (la == 1 ? n1 : n2);
      const long long r = e0 + o < noff ? e0 + o : noff - 1;
      (*HND_S(&tix[o])) = static_cast<int>(r / EL - e0 / EL);
      (*HND_S(&tix[kFO + o])) = rep(tl, nl) + nl - 1;
    }
  }
  if constexpr (TAB) {
    // the rows' columns on the axes before the last
    const int la = a.ndim - 1;
    const int EL = la == 0 ? E0 : (la == 1 ? E1 : E2);
    const long long last = (e0 + kFO < noff ? e0 + kFO : noff) - 1;
    const int nrows = static_cast<int>(last / EL - e0 / EL) + 1;
    for (int rr = tid; rr < nrows; rr += kFT) {
      const long long R = e0 / EL + rr;           // row index over the axes before the last
      const int i0 = la == 2 ? static_cast<int>(R / E1) : static_cast<int>(R);
      const int i1 = la == 2 ? static_cast<int>(R % E1) : 0;
      (*HND_S(&rtix[rr])) = rep(i0 - (n0 - 1), n0) + n0 - 1;
      (*HND_S(&rtix[kFR + rr])) = rep(i1 - (n1 - 1), n1) + n1 - 1;
    }
  }
  if constexpr (!TAB) {
    // Fourier features, phi[(ax M + m - 1) 2 + {0: sin, 1: cos}][o]
    const int M = a.num_freqs;
    for (int i = tid; i < kFO * a.ndim * M; i += kFT) {
      const int o = i % kFO, q = i / kFO, m = q % M + 1, ax = q / M;
      int t0, t1, t2;
      offset_of(o, t0, t1, t2);
      const int nax = ax == 0 ? n0 : (ax == 1 ? n1 : n2);
      const int tax = rep(ax == 0 ? t0 : (ax == 1 ? t1 : t2), nax);
      float sv, cv;
      sincospif(static_cast<float>(m) * (static_cast<float>(tax) / static_cast<float>(nax)), &sv, &cv);
      (*HND_S(&phi[(2 * (ax * M + m - 1)) * kFO + o])) = sv;
      (*HND_S(&phi[(2 * (ax * M + m - 1) + 1) * kFO + o])) = cv;
    }
  }
  __syncthreads();

  const int og = tid % 32, grp = tid / 32;
  if constexpr (TAB) {
    // hidden layer by angle addition over the last axis (see filter_table_floats)
    const int la = a.ndim - 1;
    const int EL = la == 0 ? E0 : (la == 1 ? E1 : E2);
    const long long last = (e0 + kFO < noff ? e0 + kFO : noff) - 1;
    const int nrows = static_cast<int>(last / EL - e0 / EL) + 1;
    const float* T0 = a.tab;
    const float* T1 = T0 + static_cast<long long>(HP) * E0;
    const int nn[3] = {n0, n1, n2};
    const float* Sl = a.tab + filter_trig_offset(HP, a.ndim, nn);
    const float* Cl = Sl + static_cast<long long>(HP) * EL;
    // sin A, cos A per (unit, row): A = gamma (b1 + sum of the earlier axes) + beta
    for (int i = tid; i < HP * nrows; i += kFT) {
      const int h = i / nrows, rr = i % nrows;
      float A = *HND_S(&b1[h]);
      if (la >= 1) A += __ldg(HND_G(T0 + h * E0 + (*HND_S(&rtix[rr]))));
      if (la >= 2) A += __ldg(HND_G(T1 + h * E1 + (*HND_S(&rtix[kFR + rr]))));
      if (a.gamma && h < a.hidden) A = fmaf(__ldg(HND_G(a.gamma + h)), A, __ldg(HND_G(a.beta + h)));
      float sv, cv;
      sincosf(A, &sv, &cv);
      (*HND_S(&sA[h * kFR + rr])) = sv;
      (*HND_S(&cA[h * kFR + rr])) = cv;
    }
    __syncthreads();
    // thread -> offset o (consecutive offsets read consecutive table columns),
    // units h = tid / kFO, + kFT / kFO, ...
    const int o = tid % kFO;
    const int rr = *HND_S(&tix[o]), tl = *HND_S(&tix[kFO + o]);
    for (int h = tid / kFO; h < HP; h += kFT / kFO) {
      float v = 0.f;
      if (h < a.hidden) {
        const long long j = static_cast<long long>(h) * EL + tl;
        v = fmaf(*HND_S(&sA[h * kFR + rr]), __ldg(HND_G(Cl + j)), *HND_S(&cA[h * kFR + rr]) * __ldg(HND_G(Sl + j)));
      }
      (*HND_S(&hid[h * kFO + o])) = v;
    }
  } else {
    // hidden layer: thread (og, hg) computes offsets 4 og .. 4 og + 3 x units hg HG ..
    {
      float acc[4][HG];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < HG; ++j) acc[i][j] = (*HND_S(&b1[grp * HG + j]));
      for (int f = 0; f < fin; ++f) {
        const float4 p = *HND_S(reinterpret_cast<const float4*>(phi + f * kFO + 4 * og));
        const float pv[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
        for (int j4 = 0; j4 < HG / 4; ++j4) {
          const float4 w = *HND_S(reinterpret_cast<const float4*>(w1 + f * HP + grp * HG + 4 * j4));
          const float wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) acc[i][4 * j4 + jj] = fmaf(wv[jj], pv[i], acc[i][4 * j4 + jj]);
        }
      }
      if (a.gamma) {       // per-sample feature-wise modulation of the sine layer
#pragma unroll
        for (int j = 0; j < HG; ++j) {
          const int hu = grp * HG + j;
          const float gm = hu < a.hidden ? __ldg(HND_G(a.gamma + hu)) : 0.f;
          const float bt = hu < a.hidden ? __ldg(HND_G(a.beta + hu)) : 0.f;
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[i][j] = fmaf(gm, acc[i][j], bt);
        }
      }
#pragma unroll
      for (int j = 0; j < HG; ++j)
        *HND_S(reinterpret_cast<float4*>(hid + (grp * HG + j) * kFO + 4 * og)) =
            make_float4(sine_layer(acc[0][j]), sine_layer(acc[1][j]), sine_layer(acc[2][j]), sine_layer(acc[3][j]));
    }
  }

  // output layer over the channel tiles of this CTA's group (blockIdx.y):
  // thread (og, cg) -> offsets 4 og.., channels 4 cg..
  const int cend = min(a.nc, (static_cast<int>(blockIdx.y) + 1) * a.cgroup);
  for (int ct = static_cast<int>(blockIdx.y) * a.cgroup; ct < cend; ct += kFC) {
    __syncthreads();          // hid complete / previous tile's w2 no longer read
    for (int i = tid; i < HP * kFC; i += kFT) {
      const int h = i / kFC, cc = i % kFC;
      const int c = ct + cc;
      (*HND_S(&w2[i])) = (h < a.hidden && c < a.nc) ? __ldg(HND_G(a.W2 + static_cast<long long>(a.c0 + c) * a.hidden + h)) : 0.f;
    }
    __syncthreads();
    if (a.nc - ct <= kFNarrow) {
      // narrow tile (a chunk of at most 8 channels, e.g. the large 3D grids):
      // thread -> offset tid % kFO, channels 4 (tid / kFO) .. + 3, so no
      // thread computes padding channels beyond the chunk's 8
      const int o = tid % kFO, cb = 4 * (tid / kFO);
      if (cb < a.nc - ct) {
        float acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
        for (int h = 0; h < HP; ++h) {
          const float hv = *HND_S(hid + h * kFO + o);
          const float4 wv = *HND_S(reinterpret_cast<const float4*>(w2 + h * kFC + cb));
          acc1[0] = fmaf(hv, wv.x, acc1[0]);
          acc1[1] = fmaf(hv, wv.y, acc1[1]);
          acc1[2] = fmaf(hv, wv.z, acc1[2]);
          acc1[3] = fmaf(hv, wv.w, acc1[3]);
        }
        if (e0 + o < noff) {
          const float ro = *HND_S(&rad[o]);
          const int so = *HND_S(&slot[o]);
          float kv[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int c = ct + cb + j;
            kv[j] = 0.f;
            if (c < a.nc) {
              const float bb = __ldg(HND_G(a.b2 + a.c0 + c)), al = __ldg(HND_G(a.alpha + a.c0 + c));
              kv[j] = (acc1[j] + bb) * __expf(-al * ro);
            }
          }
          store_k4(a, ct + cb, gsz, so, kv);
        }
      }
      continue;
    }
    if (a.nc - ct <= kFC / 2) {
      // half tile (9 to 16 channels left, e.g. the 128^3 grids' chunks):
      // thread -> offsets 2 (tid % 64) + {0, 1}, channels 4 (tid / 64) + {0..3}
      const int o2 = 2 * (tid % 64), cb = 4 * (tid / 64);
      float acc2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll 8
      for (int h = 0; h < HP; ++h) {
        const float2 hv = *HND_S(reinterpret_cast<const float2*>(hid + h * kFO + o2));
        const float4 wv = *HND_S(reinterpret_cast<const float4*>(w2 + h * kFC + cb));
        const float ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc2[0][j] = fmaf(hv.x, ww[j], acc2[0][j]);
          acc2[1][j] = fmaf(hv.y, ww[j], acc2[1][j]);
        }
      }
      if (cb < a.nc - ct) {
        float bb[4], al[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int c = ct + cb + j;
          bb[j] = c < a.nc ? __ldg(HND_G(a.b2 + a.c0 + c)) : 0.f;
          al[j] = c < a.nc ? __ldg(HND_G(a.alpha + a.c0 + c)) : 0.f;
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int o = o2 + i;
          if (e0 + o >= noff) continue;
          const float ro = *HND_S(&rad[o]);
          float kv[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) kv[j] = ct + cb + j < a.nc ? (acc2[i][j] + bb[j]) * __expf(-al[j] * ro) : 0.f;
          store_k4(a, ct + cb, gsz, *HND_S(&slot[o]), kv);
        }
      }
      continue;
    }
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 4
    for (int h = 0; h < HP; ++h) {
      const float4 hv = *HND_S(reinterpret_cast<const float4*>(hid + h * kFO + 4 * og));
      const float4 wv = *HND_S(reinterpret_cast<const float4*>(w2 + h * kFC + 4 * grp));
      const float hh[4] = {hv.x, hv.y, hv.z, hv.w}, ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(hh[i], ww[j], acc[i][j]);
    }
    float bb[4], al[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = ct + 4 * grp + j;
      bb[j] = c < a.nc ? __ldg(HND_G(a.b2 + a.c0 + c)) : 0.f;
      al[j] = c < a.nc ? __ldg(HND_G(a.alpha + a.c0 + c)) : 0.f;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int o = 4 * og + i;
      if (e0 + o >= noff) continue;
      const float ro = *HND_S(&rad[o]);
      float kv[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) kv[j] = ct + 4 * grp + j < a.nc ? (acc[i][j] + bb[j]) * __expf(-al[j] * ro) : 0.f;
      store_k4(a, ct + 4 * grp, gsz, *HND_S(&slot[o]), kv);
    }
  }
}

// In-place full complex forward transform of length P = 2N along one axis of
// a batch of arrays: element e of pencil (o, i) sits at (o P + e) S + i, with
// S = 2^lgS the axis stride.  Pencils are counted compactly so that ones known
// to be zero can be skipped: pencil p has o = p >> lgSc and compact inner
// index c = p & (2^lgSc - 1), mapped to i = ((c >> lgK) << lgPi) | (c & (2^lgK - 1))
// (the first 2^lgK of every 2^lgPi inner positions; lgSc = lgK = lgPi = lgS
// visits every pencil).  All extents are powers of two.
// One pencil per G lanes of the packed core; a warp takes pencils with
// consecutive i (adjacent in memory on a strided axis).  Every lane loads its
// pencil's values before the core's exchange, so the stores cannot overwrite
// unread inputs.
constexpr int kAT = 256;     // threads per CTA of the axis transform

template <int N>
struct AxisSmem {
  static constexpr size_t kBytes = Tabs<N>::kBytes + 16ull * XB<N>::kWarp * (kAT / 32);
};

struct AxisMap {
  long long npencil;
  int lgS, lgSc, lgK, lgPi;
};

template <int N>
__global__ void __launch_bounds__(kAT) k_fft_axis2(float2* __restrict__ data, const AxisMap m) {
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
  const long long stride = 1LL << m.lgS;
  for (long long p0 = static_cast<long long>(blockIdx.x) * per_cta; p0 < m.npencil;
       p0 += static_cast<long long>(gridDim.x) * per_cta) {
    const long long p = p0 + warp * PPW + pen;
    const bool act = p < m.npencil;
    const long long o = act ? p >> m.lgSc : 0;
    const long long c = act ? p & ((1LL << m.lgSc) - 1) : 0;
    const long long i = ((c >> m.lgK) << m.lgPi) | (c & ((1LL << m.lgK) - 1));
    float2* base = data + ((o * P) << m.lgS) + i;
    float2 lo[R1], hi[R1];
#pragma unroll
    for (int s = 0; s < R1; ++s) {
      const long long j = g + s * G;
      lo[s] = act ? (*HND_G(&base[j * stride])) : make_float2(0.f, 0.f);
      hi[s] = act ? (*HND_G(&base[(j + N) * stride])) : make_float2(0.f, 0.f);
    }
    cp x[R1];
    full_fwd<N>(lo, hi, x, g, buf, 0, t, 0u);
    if (act) {
#pragma unroll
      for (int s = 0; s < R1; ++s) {
        const long long kk = 2LL * spec_idx<N>(g, s);
        (*HND_G(&base[kk * stride])) = make_float2(x[s].re.x, x[s].im.x);
        (*HND_G(&base[(kk + 1) * stride])) = make_float2(x[s].re.y, x[s].im.y);
      }
    }
  }
}

}  // namespace hnd2
