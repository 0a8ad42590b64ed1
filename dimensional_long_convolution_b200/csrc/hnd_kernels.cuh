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
//   ndim 1: the column stage is a pointwise product          (k_rows1d, here)
//   ndim 2: a zero-padded 1D convolution along axis 0        (hnd_fused2.cuh, hnd_multi2.cuh)
//   ndim 3: a zero-padded 2D convolution over axes 0, 1      (hnd_multi2.cuh)
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

namespace hnd {

static __device__ const float2 g_tw[kTab] =
#include "hnd_twiddles.inc"
;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kXWarp = 4608 / 16;       // float4 per warp of exchange buffers

__device__ __forceinline__ void load_twiddles(float2* T) {
  for (int i = threadIdx.x; i < kTab; i += blockDim.x) (*HND_S(&T[i])) = g_tw[i];
}

// Shared memory of the 1D row kernel: the twiddle table and its warps' exchange buffers.
constexpr size_t kMidSmemBase = sizeof(float2) * kTab + sizeof(float4) * kXWarp * kWarps;

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
          Sa = __ldg(HND_G(sa + kk));
          Sb = __ldg(HND_G(sb + kk));
        } else {
          Sa = c_conj(__ldg(HND_G(sa + 2 * N - kk)));
          Sb = c_conj(__ldg(HND_G(sb + 2 * N - kk)));
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


// ============================================================ spectrum layout
// Problem shape as the layout code sees it.  2D and 3D spectra are converted by
// the kernels of hnd_fused2.cuh / hnd_multi2.cuh and long 1D ones by
// hnd_long1d.cuh; the kernels below serve 1D grids of at most 256 points,
// whose library order is the natural half spectrum kx in [0, n].
struct SpecDims {
  int ndim;
  int n[3];
};

__host__ __device__ __forceinline__ long long spec_per_channel(const SpecDims& d) {
  if (d.ndim == 1) return d.n[0] + 1;
  if (d.ndim == 2) return static_cast<long long>(d.n[1] + 1) * 2 * d.n[0];
  return static_cast<long long>(d.n[2] + 1) * 4 * d.n[1] * d.n[0];
}

// 1D: natural [C][n + 1] <-> library order (the same order: a copy)
static __global__ void k_spec_import(const float2* __restrict__ nat, float2* __restrict__ out, SpecDims d, long long C) {
  const long long total = spec_per_channel(d) * C;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x)
    (*HND_G(&out[e])) = (*HND_G(&nat[e]));
}

static __global__ void k_spec_export(const float2* __restrict__ lib, float2* __restrict__ nat, SpecDims d, long long C) {
  const long long total = spec_per_channel(d) * C;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x)
    (*HND_G(&nat[e])) = (*HND_G(&lib[e]));
}

// ================================================================ the filter
// 1D: the kept half [0, n] of each full padded transform (a chunk of nc
// channels of length 2n) -> library order of channels c0.., scaled.
static __global__ void k_spec_pack(const float2* __restrict__ grid, float2* __restrict__ out, SpecDims d, int c0, int nc,
                                   float scale) {
  const long long per = spec_per_channel(d);
  const long long P = 2LL * d.n[0];
  const long long total = per * nc;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long cl = e / per, o = e % per;
    (*HND_G(&out[(c0 + cl) * per + o])) = c_scale((*HND_G(&grid[cl * P + o])), scale);
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
