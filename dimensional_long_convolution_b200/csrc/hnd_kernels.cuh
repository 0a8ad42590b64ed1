// hnd_kernels.cuh -- device kernels of the gated nD linear FFT convolution
//   y[b,c,i] = q[b,c,i] * sum_j k[b,c,j] v[b,c,j] K_c[i - j]
// (HyenaND pages: blog section "HyenaND", output equation; arXiv 2607.19378
// summary, "Methodologie" (zero padding to twice the grid) and
// "Implementation: nSubQ" (forward FFT, spectral modulation, inverse FFT,
// output cropping, fused, intermediates on chip)).
//
// Common structure of every tier.  Rows along the last axis (length NL, padded
// to 2NL) are transformed two at a time: a row pair (a, b) is packed as
// z = u_a + i u_b and one complex transform serves both real rows.  The row
// stage leaves, per row pair rp and padded frequency kk in [0, 2NL), the
// packed value Zt[kk][rp].  The "column" stage, per last-axis frequency kx,
// separates the two rows' spectra from Zt[kx] and Zt[2NL - kx], convolves
// along the remaining axes, and writes back the packed inverse input
//   W[kx] = Y_a + i Y_b,   W[2NL - kx] = conj(Y_a) + i conj(Y_b).
// The inverse row stage then returns y_a + i y_b in one transform.
//   ndim 1: the column stage is a pointwise product          (k_rows1d)
//   ndim 2: a zero-padded 1D convolution along axis 0        (k_fused2d, k_mid1)
//   ndim 3: a zero-padded 2D convolution over axes 0, 1      (k_mid2, k_mid2_pair)
//
// Spectrum layouts (per channel, complex64, 1/prod(P) folded in):
//   ndim 1: natural, kx in [0, n].
//   ndim 2: n_1 column slots of 2 n_0 values in z-pencil spectral order
//           ([g][s][p] -> ky = 2 spec_index(g, s) + p).  Slot 0 holds the DC and
//           Nyquist columns combined as A = (S0 + Sn)/2 then B = (S0 - Sn)/2 (two
//           payloads), slot s >= 1 holds column kx = s.
//   ndim 3: for kx in [0, n_2], for ky in [0, 2 n_1): 2 n_0 values, same order.
#pragma once

#include "hnd_fft.cuh"
#include <cooperative_groups.h>

namespace hnd {

namespace cg = cooperative_groups;

static __device__ const float2 g_tw[kTab] =
#include "hnd_twiddles.inc"
;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kXWarp = 4608 / 16;       // float4 per warp of exchange buffers

__device__ __forceinline__ void load_twiddles(float2* T) {
  for (int i = threadIdx.x; i < kTab; i += blockDim.x) T[i] = g_tw[i];
}

// Pair ordering: consecutive blocks walk b fastest so the B samples that share
// a channel spectrum run together (the spectrum is then read from HBM once).
__device__ __forceinline__ long long pair_of(long long ord, int B, int C, int* b_out, int* c_out) {
  const int c = static_cast<int>(ord / B), b = static_cast<int>(ord % B);
  *b_out = b;
  *c_out = c;
  return static_cast<long long>(b) * C + c;
}

// Runtime twin of spec_index (used by the layout conversion kernels).
__host__ __device__ __forceinline__ int spec_index_rt(int N, int g, int s) {
  const int G = N / 8;
  const int RL = (N == 8) ? 8 : (N == 16) ? 2 : (N == 32) ? 4 : (N == 64) ? 8 : (N == 128) ? 2 : (N == 256) ? 4 : 8;
  return g + G * (s / RL) + (s % RL) * (N / RL);
}
// Padded frequency of position q in a length-2N pencil payload.
__host__ __device__ __forceinline__ int payload_freq(int N, int q) {
  const int g = q >> 4, rem = q & 15;
  return 2 * spec_index_rt(N, g, rem >> 1) + (rem & 1);
}

// ===================================================================== 2D fused
// One CTA per (b, c): rows -> columns -> inverse rows, all in shared memory.
template <int N0, int N1>
struct Fused2DSmem {
  static constexpr int RPS = N0 / 2 + 1;                    // row-pair stride (padded)
  static constexpr size_t kBytes = sizeof(float2) * (kTab + 2 * N1 * RPS) + sizeof(float4) * kXWarp * kWarps;
};

template <int N0, int N1, class IO>
__global__ void __launch_bounds__(kThreads) k_fused2d(const typename IO::T* __restrict__ q,
                                                      const typename IO::T* __restrict__ k,
                                                      const typename IO::T* __restrict__ v,
                                                      const float2* __restrict__ spec, long long sbs,
                                                      typename IO::T* __restrict__ y, int B, int C) {
  using TT = typename IO::T;
  constexpr int RPS = Fused2DSmem<N0, N1>::RPS;
  extern __shared__ float4 smem4[];
  float2* T = reinterpret_cast<float2*>(smem4);
  float2* Zb = T + kTab;
  float4* xb = reinterpret_cast<float4*>(Zb + 2 * N1 * RPS);

  load_twiddles(T);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int b, c;
  const long long pair = pair_of(blockIdx.x, B, C, &b, &c);
  constexpr long long L = static_cast<long long>(N0) * N1;
  const TT* kp = k + pair * L;
  const TT* vp = v + pair * L;
  const TT* qp = q + pair * L;
  TT* yp = y + pair * L;
  __syncthreads();

  // ---- stage 1: packed row pairs, forward padded transform along axis 1
  {
    constexpr int G = N1 / 8, PPW = 32 / G;
    const int pen = lane / G, g = lane % G;
    const unsigned mask = pencil_mask<N1>(lane);
    float4* buf = xb + warp * kXWarp + pen * XBuf<N1>::kFloat4;
    for (int rp0 = warp * PPW; rp0 < N0 / 2; rp0 += kWarps * PPW) {
      const int rp = rp0 + pen;
      const bool act = rp < N0 / 2;
      float2 x[2][8];
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const int j = g + s * G;
        const int ra = 2 * rp * N1 + j;
        x[0][s] = act ? make_float2(IO::ld(kp + ra) * IO::ld(vp + ra), IO::ld(kp + ra + N1) * IO::ld(vp + ra + N1))
                      : make_float2(0.f, 0.f);
      }
      padded_fwd<N1>(x, g, buf, T, mask);
      if (act) {
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          const int kk = 2 * spec_index<N1>(g, s);
          Zb[kk * RPS + rp] = x[0][s];
          Zb[(kk + 1) * RPS + rp] = x[1][s];
        }
      }
    }
  }
  __syncthreads();

  // ---- stage 2: per last-axis frequency, zero-padded convolution along axis 0
  {
    constexpr int G = N0 / 8, PPW = 32 / G;
    const int pen = lane / G, g = lane % G;
    const unsigned mask = pencil_mask<N0>(lane);
    float4* buf = xb + warp * kXWarp + pen * XBuf<N0>::kFloat4;
    const float2* sp = spec + static_cast<long long>(b) * sbs + static_cast<long long>(c) * (N1 + 1) * 2 * N0;
    for (int cu0 = warp * PPW; cu0 < N1; cu0 += kWarps * PPW) {
      const int cu = cu0 + pen;
      const bool act = cu < N1;
      const int kx = cu, kxm = 2 * N1 - cu;
      float2 x[2][8];
      if (cu == 0) {
        // DC and Nyquist columns (both real) combined as one complex column
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          const int i = g + s * G, rp = i >> 1;
          const float2 z0 = Zb[rp], zn = Zb[N1 * RPS + rp];
          x[0][s] = (i & 1) ? make_float2(z0.y, zn.y) : make_float2(z0.x, zn.x);
        }
        padded_fwd<N0>(x, g, buf, T, mask);
        float2 xp[2][8];
        fetch_partner<N0>(x, xp, g, buf, mask);
        const float4* A4 = reinterpret_cast<const float4*>(sp) + g * 8;
        const float4* B4 = reinterpret_cast<const float4*>(sp + 2 * N0) + g * 8;
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          const float4 a = __ldg(A4 + s), bb = __ldg(B4 + s);
          x[0][s] = c_add(c_mul(x[0][s], make_float2(a.x, a.y)), c_mul(c_conj(xp[0][s]), make_float2(bb.x, bb.y)));
          x[1][s] = c_add(c_mul(x[1][s], make_float2(a.z, a.w)), c_mul(c_conj(xp[1][s]), make_float2(bb.z, bb.w)));
        }
      } else {
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          const int i = g + s * G, rp = i >> 1;
          float2 z1 = make_float2(0.f, 0.f), z2 = z1;
          if (act) {
            z1 = Zb[kx * RPS + rp];
            z2 = Zb[kxm * RPS + rp];
          }
          x[0][s] = (i & 1) ? unpack_b(z1, z2) : unpack_a(z1, z2);
        }
        padded_fwd<N0>(x, g, buf, T, mask);
        if (act) {
          const float4* S4 = reinterpret_cast<const float4*>(sp + static_cast<long long>(cu + 1) * 2 * N0) + g * 8;
#pragma unroll
          for (int s = 0; s < 8; ++s) {
            const float4 t = __ldg(S4 + s);
            x[0][s] = c_mul(x[0][s], make_float2(t.x, t.y));
            x[1][s] = c_mul(x[1][s], make_float2(t.z, t.w));
          }
        }
      }
      padded_inv<N0>(x, g, buf, T, mask);
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const float2 own = x[0][s];
        float2 oth;
        if constexpr (G >= 2) {
          oth.x = __shfl_xor_sync(mask, own.x, 1);
          oth.y = __shfl_xor_sync(mask, own.y, 1);
        } else {
          oth = x[0][s ^ 1];
        }
        const int i = g + s * G, rp = i >> 1;
        const bool odd = i & 1;
        const float2 ya = odd ? oth : own, yb = odd ? own : oth;
        if (act) {
          if (cu == 0) {
            if (!odd) Zb[rp] = make_float2(ya.x, yb.x);
            else Zb[N1 * RPS + rp] = make_float2(ya.y, yb.y);
          } else {
            if (!odd) Zb[kx * RPS + rp] = pack_pos(ya, yb);
            else Zb[kxm * RPS + rp] = pack_neg(ya, yb);
          }
        }
      }
    }
  }
  __syncthreads();

  // ---- stage 3: inverse padded transform of row pairs, crop, output gate
  {
    constexpr int G = N1 / 8, PPW = 32 / G;
    const int pen = lane / G, g = lane % G;
    const unsigned mask = pencil_mask<N1>(lane);
    float4* buf = xb + warp * kXWarp + pen * XBuf<N1>::kFloat4;
    for (int rp0 = warp * PPW; rp0 < N0 / 2; rp0 += kWarps * PPW) {
      const int rp = rp0 + pen;
      const bool act = rp < N0 / 2;
      float2 x[2][8];
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const int kk = 2 * spec_index<N1>(g, s);
        x[0][s] = act ? Zb[kk * RPS + rp] : make_float2(0.f, 0.f);
        x[1][s] = act ? Zb[(kk + 1) * RPS + rp] : make_float2(0.f, 0.f);
      }
      padded_inv<N1>(x, g, buf, T, mask);
      if (act) {
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          const int ra = 2 * rp * N1 + g + s * G;
          IO::st(yp + ra, x[0][s].x * IO::ld(qp + ra));
          IO::st(yp + ra + N1, x[0][s].y * IO::ld(qp + ra + N1));
        }
      }
    }
  }
}

// ===================================================================== 1D fused
// Rows are independent: each warp owns row pairs, transforms, multiplies by the
// channel spectrum (natural order, kx in [0, N]) and transforms back.
template <int N, class IO, bool DUAL>
__global__ void __launch_bounds__(kThreads) k_rows1d(const typename IO::T* __restrict__ q,
                                                     const typename IO::T* __restrict__ k,
                                                     const typename IO::T* __restrict__ v,
                                                     const float2* __restrict__ spec, long long sbs,
                                                     typename IO::T* __restrict__ y, int B, int C, float sgn,
                                                     const typename IO::T* __restrict__ g2,
                                                     typename IO::T* __restrict__ y2) {
  using TT = typename IO::T;
  extern __shared__ float4 smem4[];
  float2* T = reinterpret_cast<float2*>(smem4);
  float4* xb = reinterpret_cast<float4*>(T + kTab);
  load_twiddles(T);
  __syncthreads();
  constexpr int G = N / 8, PPW = 32 / G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pen = lane / G, g = lane % G;
  const unsigned mask = pencil_mask<N>(lane);
  float4* buf = xb + warp * kXWarp + pen * XBuf<N>::kFloat4;
  const long long rows = static_cast<long long>(B) * C;
  const long long rpairs = (rows + 1) / 2;
  for (long long rp0 = (static_cast<long long>(blockIdx.x) * kWarps + warp) * PPW; rp0 < rpairs;
       rp0 += static_cast<long long>(gridDim.x) * kWarps * PPW) {
    const long long rp = rp0 + pen;
    const long long ra = 2 * rp, rb = 2 * rp + 1;
    const bool act_a = ra < rows, act_b = rb < rows;
    float2 x[2][8];
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const long long j = g + s * G;
      const float ua = act_a ? IO::ld(k + ra * N + j) * IO::ld(v + ra * N + j) : 0.f;
      const float ub = act_b ? IO::ld(k + rb * N + j) * IO::ld(v + rb * N + j) : 0.f;
      x[0][s] = make_float2(ua, ub);
    }
    padded_fwd<N>(x, g, buf, T, mask);
    float2 xp[2][8];
    fetch_partner<N>(x, xp, g, buf, mask);
    const int ba = static_cast<int>((act_a ? ra : 0) / C), ca = static_cast<int>((act_a ? ra : 0) % C);
    const int bb = static_cast<int>((act_b ? rb : 0) / C), cb = static_cast<int>((act_b ? rb : 0) % C);
    const float2* sa = spec + static_cast<long long>(ba) * sbs + static_cast<long long>(ca) * (N + 1);
    const float2* sb = spec + static_cast<long long>(bb) * sbs + static_cast<long long>(cb) * (N + 1);
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const int f = spec_index<N>(g, s);
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        const int kk = 2 * f + p;
        const float2 xa = unpack_a(x[p][s], xp[p][s]), xbv = unpack_b(x[p][s], xp[p][s]);
        float2 Sa, Sb;
        if (kk <= N) {
          Sa = __ldg(sa + kk);
          Sb = __ldg(sb + kk);
        } else {
          Sa = c_conj(__ldg(sa + 2 * N - kk));
          Sb = c_conj(__ldg(sb + 2 * N - kk));
        }
        Sa.y *= sgn, Sb.y *= sgn;     // sgn = -1: conjugate spectrum (adjoint)
        x[p][s] = pack_pos(c_mul(xa, Sa), c_mul(xbv, Sb));
      }
    }
    padded_inv<N>(x, g, buf, T, mask);
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const long long j = g + s * G;
      if (act_a) IO::st(y + ra * N + j, x[0][s].x * IO::ld(q + ra * N + j));
      if (act_b) IO::st(y + rb * N + j, x[0][s].y * IO::ld(q + rb * N + j));
      if constexpr (DUAL) {       // second gated output of the same convolution
        if (act_a) IO::st(y2 + ra * N + j, x[0][s].x * IO::ld(g2 + ra * N + j));
        if (act_b) IO::st(y2 + rb * N + j, x[0][s].y * IO::ld(g2 + rb * N + j));
      }
    }
  }
}

// ============================================================ multi-pass rows
// Workspace of one wave: Zt[wp][kk][rp], wp = pair within the wave,
// kk in [0, 2 NL), rp in [0, R/2) with R = rows per volume.
template <int NL>
struct RowTile {
  static constexpr int RPB = (4096 / NL) < 32 ? (4096 / NL) : 32;   // row pairs per CTA
  static constexpr int TS = RPB + 1;                                 // padded tile stride
  static constexpr size_t kBytes = sizeof(float2) * (kTab + 2 * NL * TS) + sizeof(float4) * kXWarp * kWarps;
};

template <int NL, class IO>
__global__ void __launch_bounds__(kThreads) k_rowfwd(const typename IO::T* __restrict__ k,
                                                     const typename IO::T* __restrict__ v,
                                                     float2* __restrict__ Zt, long long ord0, int rp_total,
                                                     int B, int C) {
  using TT = typename IO::T;
  constexpr int RPB = RowTile<NL>::RPB, TS = RowTile<NL>::TS;
  extern __shared__ float4 smem4[];
  float2* T = reinterpret_cast<float2*>(smem4);
  float2* tile = T + kTab;
  float4* xb = reinterpret_cast<float4*>(tile + 2 * NL * TS);
  load_twiddles(T);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int b, c;
  const long long pair = pair_of(ord0 + blockIdx.x, B, C, &b, &c);
  const long long L = static_cast<long long>(rp_total) * 2 * NL;
  const TT* kp = k + pair * L;
  const TT* vp = v + pair * L;
  const int rpb = blockIdx.y * RPB;
  const int nrp = min(RPB, rp_total - rpb);
  __syncthreads();
  constexpr int G = NL / 8, PPW = 32 / G;
  const int pen = lane / G, g = lane % G;
  const unsigned mask = pencil_mask<NL>(lane);
  float4* buf = xb + warp * kXWarp + pen * XBuf<NL>::kFloat4;
  for (int r0 = warp * PPW; r0 < RPB; r0 += kWarps * PPW) {
    const int rl = r0 + pen;
    const bool act = rl < nrp;
    const long long row = 2LL * (rpb + rl);
    float2 x[2][8];
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const long long ra = row * NL + g + s * G;
      x[0][s] = act ? make_float2(IO::ld(kp + ra) * IO::ld(vp + ra), IO::ld(kp + ra + NL) * IO::ld(vp + ra + NL))
                    : make_float2(0.f, 0.f);
    }
    padded_fwd<NL>(x, g, buf, T, mask);
    if (rl < RPB) {
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const int kk = 2 * spec_index<NL>(g, s);
        tile[kk * TS + rl] = x[0][s];
        tile[(kk + 1) * TS + rl] = x[1][s];
      }
    }
  }
  __syncthreads();
  float2* zt = Zt + static_cast<long long>(blockIdx.x) * 2 * NL * rp_total;
  for (int e = threadIdx.x; e < 2 * NL * RPB; e += kThreads) {
    const int kk = e / RPB, rl = e % RPB;
    if (rl < nrp) zt[static_cast<long long>(kk) * rp_total + rpb + rl] = tile[kk * TS + rl];
  }
}

template <int NL, class IO>
__global__ void __launch_bounds__(kThreads) k_rowinv(const float2* __restrict__ Zt,
                                                     const typename IO::T* __restrict__ q,
                                                     typename IO::T* __restrict__ y, long long ord0, int rp_total,
                                                     int B, int C) {
  using TT = typename IO::T;
  constexpr int RPB = RowTile<NL>::RPB, TS = RowTile<NL>::TS;
  extern __shared__ float4 smem4[];
  float2* T = reinterpret_cast<float2*>(smem4);
  float2* tile = T + kTab;
  float4* xb = reinterpret_cast<float4*>(tile + 2 * NL * TS);
  load_twiddles(T);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int b, c;
  const long long pair = pair_of(ord0 + blockIdx.x, B, C, &b, &c);
  const long long L = static_cast<long long>(rp_total) * 2 * NL;
  const TT* qp = q + pair * L;
  TT* yp = y + pair * L;
  const int rpb = blockIdx.y * RPB;
  const int nrp = min(RPB, rp_total - rpb);
  const float2* zt = Zt + static_cast<long long>(blockIdx.x) * 2 * NL * rp_total;
  for (int e = threadIdx.x; e < 2 * NL * RPB; e += kThreads) {
    const int kk = e / RPB, rl = e % RPB;
    tile[kk * TS + rl] = (rl < nrp) ? zt[static_cast<long long>(kk) * rp_total + rpb + rl] : make_float2(0.f, 0.f);
  }
  __syncthreads();
  constexpr int G = NL / 8, PPW = 32 / G;
  const int pen = lane / G, g = lane % G;
  const unsigned mask = pencil_mask<NL>(lane);
  float4* buf = xb + warp * kXWarp + pen * XBuf<NL>::kFloat4;
  for (int r0 = warp * PPW; r0 < RPB; r0 += kWarps * PPW) {
    const int rl = r0 + pen;
    const bool act = rl < nrp;
    float2 x[2][8];
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const int kk = 2 * spec_index<NL>(g, s);
      x[0][s] = (rl < RPB) ? tile[kk * TS + rl] : make_float2(0.f, 0.f);
      x[1][s] = (rl < RPB) ? tile[(kk + 1) * TS + rl] : make_float2(0.f, 0.f);
    }
    padded_inv<NL>(x, g, buf, T, mask);
    if (act) {
      const long long row = 2LL * (rpb + rl);
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const long long ra = row * NL + g + s * G;
        IO::st(yp + ra, x[0][s].x * IO::ld(qp + ra));
        IO::st(yp + ra + NL, x[0][s].y * IO::ld(qp + ra + NL));
      }
    }
  }
}

// ================================================================ 2D columns
// Multi-pass column stage of a 2D problem: one pencil per column unit.
constexpr size_t kMidSmemBase = sizeof(float2) * kTab + sizeof(float4) * kXWarp * kWarps;

template <int N0>
__global__ void __launch_bounds__(kThreads) k_mid1(float2* __restrict__ Zt, const float2* __restrict__ spec,
                                                   long long sbs, int N1, long long ord0, int B, int C) {
  extern __shared__ float4 smem4[];
  float2* T = reinterpret_cast<float2*>(smem4);
  float4* xb = reinterpret_cast<float4*>(T + kTab);
  load_twiddles(T);
  __syncthreads();
  constexpr int G = N0 / 8, PPW = 32 / G, RP = N0 / 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pen = lane / G, g = lane % G;
  const unsigned mask = pencil_mask<N0>(lane);
  float4* buf = xb + warp * kXWarp + pen * XBuf<N0>::kFloat4;
  int b, c;
  pair_of(ord0 + blockIdx.x, B, C, &b, &c);
  float2* zt = Zt + static_cast<long long>(blockIdx.x) * 2 * N1 * RP;
  const float2* sp = spec + static_cast<long long>(b) * sbs + static_cast<long long>(c) * (N1 + 1) * 2 * N0;
  const int cu = (blockIdx.y * kWarps + warp) * PPW + pen;
  const bool act = cu < N1;
  const int kx = act ? cu : 1, kxm = 2 * N1 - kx;
  float2 x[2][8];
  if (cu == 0) {
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const int i = g + s * G, rp = i >> 1;
      const float2 z0 = zt[rp], zn = zt[static_cast<long long>(N1) * RP + rp];
      x[0][s] = (i & 1) ? make_float2(z0.y, zn.y) : make_float2(z0.x, zn.x);
    }
    padded_fwd<N0>(x, g, buf, T, mask);
    float2 xp[2][8];
    fetch_partner<N0>(x, xp, g, buf, mask);
    const float4* A4 = reinterpret_cast<const float4*>(sp) + g * 8;
    const float4* B4 = reinterpret_cast<const float4*>(sp + 2 * N0) + g * 8;
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const float4 a = __ldg(A4 + s), bb = __ldg(B4 + s);
      x[0][s] = c_add(c_mul(x[0][s], make_float2(a.x, a.y)), c_mul(c_conj(xp[0][s]), make_float2(bb.x, bb.y)));
      x[1][s] = c_add(c_mul(x[1][s], make_float2(a.z, a.w)), c_mul(c_conj(xp[1][s]), make_float2(bb.z, bb.w)));
    }
  } else {
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const int i = g + s * G, rp = i >> 1;
      float2 z1 = make_float2(0.f, 0.f), z2 = z1;
      if (act) {
        z1 = zt[static_cast<long long>(kx) * RP + rp];
        z2 = zt[static_cast<long long>(kxm) * RP + rp];
      }
      x[0][s] = (i & 1) ? unpack_b(z1, z2) : unpack_a(z1, z2);
    }
    padded_fwd<N0>(x, g, buf, T, mask);
    if (act) {
      const float4* S4 = reinterpret_cast<const float4*>(sp + static_cast<long long>(cu + 1) * 2 * N0) + g * 8;
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const float4 t = __ldg(S4 + s);
        x[0][s] = c_mul(x[0][s], make_float2(t.x, t.y));
        x[1][s] = c_mul(x[1][s], make_float2(t.z, t.w));
      }
    }
  }
  padded_inv<N0>(x, g, buf, T, mask);
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const float2 own = x[0][s];
    float2 oth;
    if constexpr (G >= 2) {
      oth.x = __shfl_xor_sync(mask, own.x, 1);
      oth.y = __shfl_xor_sync(mask, own.y, 1);
    } else {
      oth = x[0][s ^ 1];
    }
    const int i = g + s * G, rp = i >> 1;
    const bool odd = i & 1;
    const float2 ya = odd ? oth : own, yb = odd ? own : oth;
    if (act) {
      if (cu == 0) {
        if (!odd) zt[rp] = make_float2(ya.x, yb.x);
        else zt[static_cast<long long>(N1) * RP + rp] = make_float2(ya.y, yb.y);
      } else {
        if (!odd) zt[static_cast<long long>(kx) * RP + rp] = pack_pos(ya, yb);
        else zt[static_cast<long long>(kxm) * RP + rp] = pack_neg(ya, yb);
      }
    }
  }
}

// ================================================================= 3D slabs
// For one last-axis frequency kx: the (axis 0, axis 1) slab of both packed
// rows' spectra, zero-padded 2D convolution with the channel's slab spectrum
// S[kz][ky][kx], written back packed.  Steps: y transform per z, z-pencil
// convolution per ky, inverse y transform per z.
template <int N0, int N1>
struct SlabSmem {
  static constexpr int FS = N0 + 1;                         // padded z stride
  static constexpr size_t kBytes = kMidSmemBase + sizeof(float2) * 2 * N1 * FS;
  static constexpr size_t kHalfBytes = kMidSmemBase + sizeof(float2) * N1 * FS;
};

template <int N0, int N1>
__device__ __forceinline__ void slab_load_rows(const float2* __restrict__ zt, long long RPn, int kx, int kxm,
                                               bool self_conj, int z, int g, float2 (&x)[2][8]) {
  constexpr int G = N1 / 8;
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const int yy = g + s * G;
    const long long i = static_cast<long long>(z) * N1 + yy, rp = i >> 1;
    const float2 z1 = zt[kx * RPn + rp];
    const float2 z2 = self_conj ? z1 : zt[kxm * RPn + rp];
    x[0][s] = (yy & 1) ? unpack_b(z1, z2) : unpack_a(z1, z2);
  }
}

template <int N0, int N1>
__device__ __forceinline__ void slab_store_rows(float2* __restrict__ zt, long long RPn, int kx, int kxm,
                                                bool self_conj, int z, int g, unsigned mask, float2 (&x)[2][8]) {
  constexpr int G = N1 / 8;
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const float2 own = x[0][s];
    float2 oth;
    if constexpr (G >= 2) {
      oth.x = __shfl_xor_sync(mask, own.x, 1);
      oth.y = __shfl_xor_sync(mask, own.y, 1);
    } else {
      oth = x[0][s ^ 1];
    }
    const int yy = g + s * G;
    const long long i = static_cast<long long>(z) * N1 + yy, rp = i >> 1;
    const bool odd = yy & 1;
    const float2 ya = odd ? oth : own, yb = odd ? own : oth;
    if (self_conj) {
      if (!odd) zt[kx * RPn + rp] = make_float2(ya.x, yb.x);
    } else {
      if (!odd) zt[kx * RPn + rp] = pack_pos(ya, yb);
      else zt[kxm * RPn + rp] = pack_neg(ya, yb);
    }
  }
}

// z-pencil convolution for padded y-frequencies ky handled by this CTA.
// F holds [kyl][z] (stride FS); ky = ky_of(kyl).
template <int N0>
__device__ __forceinline__ void slab_zconv(float2* F, int FS, int nky, int ky_mul, int ky_add,
                                           const float2* __restrict__ sslab, const float2* T, float4* xb) {
  constexpr int G = N0 / 8, PPW = 32 / G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pen = lane / G, g = lane % G;
  const unsigned mask = pencil_mask<N0>(lane);
  float4* buf = xb + warp * kXWarp + pen * XBuf<N0>::kFloat4;
  for (int k0 = warp * PPW; k0 < nky; k0 += kWarps * PPW) {
    const int kyl = k0 + pen;
    const bool act = kyl < nky;
    float2 x[2][8];
#pragma unroll
    for (int s = 0; s < 8; ++s) x[0][s] = act ? F[kyl * FS + g + s * G] : make_float2(0.f, 0.f);
    padded_fwd<N0>(x, g, buf, T, mask);
    if (act) {
      const int ky = kyl * ky_mul + ky_add;
      const float4* S4 = reinterpret_cast<const float4*>(sslab + static_cast<long long>(ky) * 2 * N0) + g * 8;
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const float4 t = __ldg(S4 + s);
        x[0][s] = c_mul(x[0][s], make_float2(t.x, t.y));
        x[1][s] = c_mul(x[1][s], make_float2(t.z, t.w));
      }
    }
    padded_inv<N0>(x, g, buf, T, mask);
    if (act) {
#pragma unroll
      for (int s = 0; s < 8; ++s) F[kyl * FS + g + s * G] = x[0][s];
    }
  }
}

template <int N0, int N1>
__global__ void __launch_bounds__(kThreads) k_mid2(float2* __restrict__ Zt, const float2* __restrict__ spec,
                                                   long long sbs, int N2, long long ord0, int B, int C) {
  constexpr int FS = SlabSmem<N0, N1>::FS;
  extern __shared__ float4 smem4[];
  float2* T = reinterpret_cast<float2*>(smem4);
  float4* xb = reinterpret_cast<float4*>(T + kTab);
  float2* F = reinterpret_cast<float2*>(xb + kXWarp * kWarps);    // [2 N1][FS]
  load_twiddles(T);
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int b, c;
  pair_of(ord0 + blockIdx.x, B, C, &b, &c);
  const long long RPn = static_cast<long long>(N0) * N1 / 2;
  float2* zt = Zt + static_cast<long long>(blockIdx.x) * 2 * N2 * RPn;
  const int kx = blockIdx.y;
  const bool self_conj = (kx == 0) || (kx == N2);
  const int kxm = self_conj ? kx : 2 * N2 - kx;
  const long long slab = 4LL * N1 * N0;
  const float2* sslab = spec + static_cast<long long>(b) * sbs + static_cast<long long>(c) * (N2 + 1) * slab +
                        static_cast<long long>(kx) * slab;
  // step 1: y transforms, one pencil per z
  {
    constexpr int G = N1 / 8, PPW = 32 / G;
    const int pen = lane / G, g = lane % G;
    const unsigned mask = pencil_mask<N1>(lane);
    float4* buf = xb + warp * kXWarp + pen * XBuf<N1>::kFloat4;
    for (int z0 = warp * PPW; z0 < N0; z0 += kWarps * PPW) {
      const int z = z0 + pen;
      const bool act = z < N0;
      float2 x[2][8];
      if (act) slab_load_rows<N0, N1>(zt, RPn, kx, kxm, self_conj, z, g, x);
      else {
#pragma unroll
        for (int s = 0; s < 8; ++s) x[0][s] = make_float2(0.f, 0.f);
      }
      padded_fwd<N1>(x, g, buf, T, mask);
      if (act) {
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          const int ky = 2 * spec_index<N1>(g, s);
          F[ky * FS + z] = x[0][s];
          F[(ky + 1) * FS + z] = x[1][s];
        }
      }
    }
  }
  __syncthreads();
  // step 2: z-pencil convolutions
  slab_zconv<N0>(F, FS, 2 * N1, 1, 0, sslab, T, xb);
  __syncthreads();
  // step 3: inverse y transforms, write back packed
  {
    constexpr int G = N1 / 8, PPW = 32 / G;
    const int pen = lane / G, g = lane % G;
    const unsigned mask = pencil_mask<N1>(lane);
    float4* buf = xb + warp * kXWarp + pen * XBuf<N1>::kFloat4;
    for (int z0 = warp * PPW; z0 < N0; z0 += kWarps * PPW) {
      const int z = z0 + pen;
      const bool act = z < N0;
      float2 x[2][8];
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const int ky = 2 * spec_index<N1>(g, s);
        x[0][s] = act ? F[ky * FS + z] : make_float2(0.f, 0.f);
        x[1][s] = act ? F[(ky + 1) * FS + z] : make_float2(0.f, 0.f);
      }
      padded_inv<N1>(x, g, buf, T, mask);
      if (act) slab_store_rows<N0, N1>(zt, RPn, kx, kxm, self_conj, z, g, mask, x);
    }
  }
}

// Two-CTA cluster version for slabs too large for one CTA: CTA h keeps the
// y-frequencies of parity h (ky = 2m + h), so each holds half of the padded
// slab.  The inverse y transform of row z needs both halves: CTA h finishes
// rows z in [h N0/2, (h+1) N0/2) reading the other half through distributed
// shared memory.
template <int N0, int N1>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads)
    k_mid2_pair(float2* __restrict__ Zt, const float2* __restrict__ spec, long long sbs, int N2, long long ord0,
                int B, int C) {
  constexpr int FS = SlabSmem<N0, N1>::FS;
  extern __shared__ float4 smem4[];
  float2* T = reinterpret_cast<float2*>(smem4);
  float4* xb = reinterpret_cast<float4*>(T + kTab);
  float2* F = reinterpret_cast<float2*>(xb + kXWarp * kWarps);    // [N1][FS], this CTA's parity
  cg::cluster_group cluster = cg::this_cluster();
  const int h = static_cast<int>(cluster.block_rank());
  float2* Fo = cluster.map_shared_rank(F, h ^ 1);
  load_twiddles(T);
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int b, c;
  pair_of(ord0 + blockIdx.x / 2, B, C, &b, &c);
  const long long RPn = static_cast<long long>(N0) * N1 / 2;
  float2* zt = Zt + static_cast<long long>(blockIdx.x / 2) * 2 * N2 * RPn;
  const int kx = blockIdx.y;
  const bool self_conj = (kx == 0) || (kx == N2);
  const int kxm = self_conj ? kx : 2 * N2 - kx;
  const long long slab = 4LL * N1 * N0;
  const float2* sslab = spec + static_cast<long long>(b) * sbs + static_cast<long long>(c) * (N2 + 1) * slab +
                        static_cast<long long>(kx) * slab;
  {
    constexpr int G = N1 / 8, PPW = 32 / G;
    const int pen = lane / G, g = lane % G;
    const unsigned mask = pencil_mask<N1>(lane);
    float4* buf = xb + warp * kXWarp + pen * XBuf<N1>::kFloat4;
    for (int z0 = warp * PPW; z0 < N0; z0 += kWarps * PPW) {
      const int z = z0 + pen;
      const bool act = z < N0;
      float2 x[2][8];
      if (act) slab_load_rows<N0, N1>(zt, RPn, kx, kxm, self_conj, z, g, x);
      else {
#pragma unroll
        for (int s = 0; s < 8; ++s) x[0][s] = make_float2(0.f, 0.f);
      }
      padded_fwd<N1>(x, g, buf, T, mask);
      if (act) {
#pragma unroll
        for (int s = 0; s < 8; ++s) F[spec_index<N1>(g, s) * FS + z] = x[h][s];
      }
    }
  }
  __syncthreads();
  slab_zconv<N0>(F, FS, N1, 2, h, sslab, T, xb);
  cluster.sync();
  {
    constexpr int G = N1 / 8, PPW = 32 / G;
    const int pen = lane / G, g = lane % G;
    const unsigned mask = pencil_mask<N1>(lane);
    float4* buf = xb + warp * kXWarp + pen * XBuf<N1>::kFloat4;
    const float2* Fe = h == 0 ? F : Fo;
    const float2* Fd = h == 0 ? Fo : F;
    for (int z0 = warp * PPW; z0 < N0 / 2; z0 += kWarps * PPW) {
      const int z = h * (N0 / 2) + z0 + pen;
      const bool act = z0 + pen < N0 / 2;
      float2 x[2][8];
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const int m = spec_index<N1>(g, s);
        x[0][s] = act ? Fe[m * FS + z] : make_float2(0.f, 0.f);
        x[1][s] = act ? Fd[m * FS + z] : make_float2(0.f, 0.f);
      }
      padded_inv<N1>(x, g, buf, T, mask);
      if (act) slab_store_rows<N0, N1>(zt, RPn, kx, kxm, self_conj, z, g, mask, x);
    }
  }
  cluster.sync();
}

// ============================================================ spectrum layout
// Natural half-spectrum index (flattened [P_0..P_{d-2}, n_last + 1]) of the
// library-order position o within one channel; for the 2D combined slot the
// A payload positions report kind 1 and B positions kind 2.
struct SpecDims {
  int ndim;
  int n[3];
};

__host__ __device__ __forceinline__ long long spec_per_channel(const SpecDims& d) {
  if (d.ndim == 1) return d.n[0] + 1;
  if (d.ndim == 2) return static_cast<long long>(d.n[1] + 1) * 2 * d.n[0];
  return static_cast<long long>(d.n[2] + 1) * 4 * d.n[1] * d.n[0];
}

// Returns natural index; kind: 0 plain, 1 = A (also fills nat2 = Nyquist index), 2 = B.
__device__ __forceinline__ long long spec_natural(const SpecDims& d, long long o, int* kind, long long* nat2) {
  *kind = 0;
  if (d.ndim == 1) return o;
  if (d.ndim == 2) {
    const int N0 = d.n[0], N1 = d.n[1];
    const int W = N1 + 1;
    if (o < 4LL * N0) {
      const int part = static_cast<int>(o / (2 * N0));
      const int ky = payload_freq(N0, static_cast<int>(o % (2 * N0)));
      *kind = 1 + part;
      *nat2 = static_cast<long long>(ky) * W + N1;
      return static_cast<long long>(ky) * W;
    }
    const long long r = o - 4LL * N0;
    const int kx = static_cast<int>(r / (2 * N0)) + 1;
    const int ky = payload_freq(N0, static_cast<int>(r % (2 * N0)));
    return static_cast<long long>(ky) * W + kx;
  }
  const int N0 = d.n[0], N1 = d.n[1], N2 = d.n[2];
  const long long slab = 4LL * N1 * N0;
  const int kx = static_cast<int>(o / slab);
  const long long r = o % slab;
  const int ky = static_cast<int>(r / (2 * N0));
  const int kz = payload_freq(N0, static_cast<int>(r % (2 * N0)));
  return (static_cast<long long>(kz) * (2 * N1) + ky) * (N2 + 1) + kx;
}

// natural [C][half] -> library order
static __global__ void k_spec_import(const float2* __restrict__ nat, float2* __restrict__ out, SpecDims d, long long C) {
  const long long per = spec_per_channel(d);
  const long long total = per * C;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long c = e / per, o = e % per;
    int kind;
    long long n2 = 0;
    const long long n1 = spec_natural(d, o, &kind, &n2);
    const float2* src = nat + c * per;
    float2 val;
    if (kind == 0) {
      val = src[n1];
    } else {
      // A at the DC slot, B at the Nyquist slot of the same ky
      const float2 s0 = src[n1], sn = src[n2];
      val = (kind == 1) ? c_scale(c_add(s0, sn), 0.5f) : c_scale(c_sub(s0, sn), 0.5f);
    }
    out[e] = val;
  }
}

// library order -> natural [C][half]
static __global__ void k_spec_export(const float2* __restrict__ lib, float2* __restrict__ nat, SpecDims d, long long C) {
  const long long per = spec_per_channel(d);
  const long long total = per * C;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long c = e / per, o = e % per;
    int kind;
    long long n2 = 0;
    const long long n1 = spec_natural(d, o, &kind, &n2);
    float2* dst = nat + c * per;
    if (kind == 0) {
      dst[n1] = lib[e];
    } else if (kind == 1) {
      // the A position of slot 0 rebuilds both the DC and Nyquist entries
      const float2 a = lib[e], bb = lib[e + 2 * d.n[0]];
      dst[n1] = c_add(a, bb);
      dst[n2] = c_sub(a, bb);
    }
  }
}

// ================================================================ the filter
// Full-grid natural spectra (chunk of channels) -> library order, scaled.
static __global__ void k_spec_pack(const float2* __restrict__ grid, float2* __restrict__ out, SpecDims d, int c0, int nc,
                            float scale) {
  const long long per = spec_per_channel(d);
  const long long total = per * nc;
  int P[3] = {1, 1, 1};
  long long gsz = 1;
  for (int a = 0; a < d.ndim; ++a) {
    P[a] = 2 * d.n[a];
    gsz *= P[a];
  }
  const int last = d.ndim - 1;
  const int W = d.n[last] + 1;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long cl = e / per, o = e % per;
    int kind;
    long long n2 = 0;
    const long long n1 = spec_natural(d, o, &kind, &n2);
    // half index -> full-grid index (the last axis keeps [0, n_last])
    auto full = [&](long long h) { return (h / W) * P[last] + (h % W); };
    const float2* src = grid + cl * gsz;
    float2 val;
    if (kind == 0) {
      val = src[full(n1)];
    } else {
      const float2 s0 = src[full(n1)], sn = src[full(n2)];
      val = (kind == 1) ? c_scale(c_add(s0, sn), 0.5f) : c_scale(c_sub(s0, sn), 0.5f);
    }
    out[(c0 + cl) * per + o] = c_scale(val, scale);
  }
}

// ================================================================ diagnostics
// Waits on a flag nothing sets, with an iteration and clock limit; records a
// timeout in the status word and returns.
// Both limits end the loop: the clock limit in normal operation, the
// iteration cap (each iteration sleeps up to about 2 us) as a backstop.
static __global__ void k_bounded_wait(int* status, const volatile int* flag, long long limit_cycles, long long max_it) {
  if (threadIdx.x != 0) return;
  const long long t0 = clock64();
  for (long long it = 0; it < max_it; ++it) {
    if (*flag != 0) return;
    if (clock64() - t0 > limit_cycles) break;
    __nanosleep(1000);
  }
  set_status(status, 6 /* HYENA_ND_ERR_DEVICE_TIMEOUT */);
}

}  // namespace hnd
