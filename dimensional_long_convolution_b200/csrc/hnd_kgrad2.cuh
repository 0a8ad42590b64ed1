// hnd_kgrad2.cuh -- the kernel-value gradient on the 2D multi-pass tier,
//   dK[c, t] = sum_b sum_{i in [0,n)^2} z[b,c,i] u[b,c,i - t],   z = q dy, u = k v,
// for every offset t in [-(n_0-1), n_0-1] x [-(n_1-1), n_1-1] (blog "Native
// multi-dimensional subquadratic operators via input-dependent long
// convolutions", gradient sections: the kernel gradient by correlation),
// through the forward's row-pair and half-spectrum stages instead of full
// complex grids:
//   forward rows   k_rowfwd2 on u and on z: packed row spectra Zt_u, Zt_z of
//                  every volume of a wave of channels (rows r and r + n0/2
//                  share one complex transform)
//   k_kgcol        per last-axis frequency kx in [0, n1] and channel: the
//                  padded column transforms U_b, Z_b of every sample, the sum
//                  A = sum_b Z_b conj(U_b) in fixed b order (deterministic),
//                  and the full-length inverse column transform (all 2 n0
//                  rows: every offset t0 is needed), stored as packed row
//                  pairs (s0, s0 + n0) of the channel's offset grid
//   k_kginv        full-length inverse row transforms of those pairs (the
//                  real and imaginary parts are the two rows), read out at the
//                  offsets t (slot t mod 2n) with the 1 / prod(P) scale
// On the 2n grid the correlation does not alias, so slot t mod 2n of the
// inverse of A is exactly dK[t]; slots n0 and n1 (offset +-n) are never read.
// A column unit runs on two pencils of a warp: pencil 0 transforms u's
// column, pencil 1 z's, and the two trade halves of their spectra by warp
// shuffles to form the product, each accumulating half of the slots.  The
// combined DC/Nyquist unit (kx = 0 and kx = n1, both real columns; its own
// launch, k_kgcol_dc) transforms u + i z of the DC column on pencil 0 and of
// the Nyquist column on pencil 1, and separates U and Z with the partner
// frequency -k.
#pragma once

#include "hnd_long1d.cuh"
#include "hnd_multi2.cuh"

namespace hnd2 {

template <int N0>
struct KGC {
  static constexpr int G = P2<N0>::G, PPW = 32 / G, R1 = P2<N0>::R1, HS = R1 / 2, H = R1 / 2;
  static constexpr int UPW = PPW / 2;                    // column units per warp (two pencils each)
  static constexpr int UPB = kWM * UPW;                  // units per CTA
  static constexpr size_t kBytes = Tabs<N0>::kBytes + 16ull * XB<N0>::kWarp * kWM;
};

// z conj(u) per path
__device__ __forceinline__ cp cmul_conj(cp z, cp u) {
  return {pfma(z.im, u.im, pmul(z.re, u.re)), pfma(z.im, u.re, pmul(make_float2(-z.re.x, -z.re.y), u.im))};
}

__device__ __forceinline__ cp shfl_cp(cp v, int lanemask) {
  cp r;
  r.re.x = __shfl_xor_sync(0xffffffffu, v.re.x, lanemask);
  r.re.y = __shfl_xor_sync(0xffffffffu, v.re.y, lanemask);
  r.im.x = __shfl_xor_sync(0xffffffffu, v.im.x, lanemask);
  r.im.y = __shfl_xor_sync(0xffffffffu, v.im.y, lanemask);
  return r;
}

// The column of unit cu (kx, partner kxm) of one volume's packed row spectra,
// unpacked into the natural order of the padded column transform (rows
// [0, n0/2) from the first rows of the pairs, [n0/2, n0) from the second).
template <int N0>
__device__ __forceinline__ void kg_column_in(const float2* __restrict__ zt, int N1, int kx, int kxm, int g,
                                             float2 (&z)[P2<N0>::R1]) {
  constexpr int G = P2<N0>::G, RP = N0 / 2, HS = P2<N0>::R1 / 2;
#pragma unroll
  for (int s = 0; s < HS; ++s) {
    const int rp = g + s * G;
    const float2 z1 = zt_ld(zt + static_cast<long long>(kx) * RP + rp);
    const float2 z2 = zt_ld(zt + static_cast<long long>(kxm) * RP + rp);
    z[s] = unpack_a(z1, z2);
    z[s + HS] = unpack_b(z1, z2);
  }
}

// Packed row pairs (s0, s0 + n0) of the channel's offset grid at column unit
// cu from the full inverse column transform: lo[s] = row g + s G, hi[s] = row
// g + s G + n0.
template <int N0>
__device__ __forceinline__ void kg_column_out(float2* __restrict__ zk, int N1, int cu, int g,
                                              const float2 (&lo)[P2<N0>::R1], const float2 (&hi)[P2<N0>::R1]) {
  constexpr int G = P2<N0>::G, R1 = P2<N0>::R1;
#pragma unroll
  for (int s = 0; s < R1; ++s) {
    const int s0 = g + s * G;
    if (cu == 0) {          // DC + i Nyquist: both columns real
      zt_st(zk + s0, make_float2(lo[s].x, hi[s].x));
      zt_st(zk + static_cast<long long>(N1) * N0 + s0, make_float2(lo[s].y, hi[s].y));
    } else {
      zt_st(zk + static_cast<long long>(cu) * N0 + s0, pack_pos(lo[s], hi[s]));
      zt_st(zk + static_cast<long long>(2 * N1 - cu) * N0 + s0, pack_neg(lo[s], hi[s]));
    }
  }
}

// General unit cu >= 1: pencil 0 (role 0) holds U, pencil 1 Z; role 0
// accumulates slots [0, H), role 1 slots [H, R1).
template <int N0>
__device__ __forceinline__ void kgcol_general(const Tabs<N0> t, float4* buf, const float2* __restrict__ zu,
                                              const float2* __restrict__ zz, long long zvol, float2* __restrict__ zk,
                                              int N1, int B, int cu, int role, int g) {
  using K = KGC<N0>;
  constexpr int R1 = K::R1, H = K::H, G = K::G;
  const bool act = cu < N1;
  const int kx = act ? cu : 1, kxm = 2 * N1 - kx;
  cp acc[H];
#pragma unroll
  for (int j = 0; j < H; ++j) acc[j] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  for (int b = 0; b < B; ++b) {
    float2 in[R1];
    kg_column_in<N0>((role == 0 ? zu : zz) + b * zvol, N1, kx, kxm, g, in);
    cp x[R1];
    padded_fwd<N0>(in, x, g, buf, 0, t, 0u);
#pragma unroll
    for (int j = 0; j < H; ++j) {
      const cp mine = role == 0 ? x[j] : x[j + H];
      const cp other = shfl_cp(role == 0 ? x[j + H] : x[j], G);
      const cp u = role == 0 ? mine : other, z = role == 0 ? other : mine;
      const cp p = cmul_conj(z, u);
      acc[j] = cadd(acc[j], p);
    }
  }
  // pencil 0 gathers the other half of the slots and runs the inverse (pencil 1
  // runs the same code on a copy and does not store)
  cp a[R1];
#pragma unroll
  for (int j = 0; j < H; ++j) {
    const cp other = shfl_cp(acc[j], G);
    a[j] = role == 0 ? acc[j] : other;
    a[j + H] = role == 0 ? other : acc[j];
  }
  float2 lo[R1], hi[R1];
  l1_full_inv<N0>(a, lo, hi, g, buf, t);
  if (act && role == 0) kg_column_out<N0>(zk, N1, cu, g, lo, hi);
}

// The combined DC/Nyquist unit: role 0 transforms w = u + i z of the DC
// column, role 1 of the Nyquist column (all four are real columns); with Wm
// the transform at -k, U = (W + conj Wm) / 2 and Z = (W - conj Wm) / (2i), so
//   Z conj(U) = Im(W Wm) / 2 - i (|W|^2 - |Wm|^2) / 4.
// Role 0 ends with A_DC, role 1 with A_Nyq; the inverse input is A_DC + i A_Nyq.
template <int N0>
__device__ __forceinline__ void kgcol_dc_nyquist(const Tabs<N0> t, float4* buf, const float2* __restrict__ zu,
                                                 const float2* __restrict__ zz, long long zvol,
                                                 float2* __restrict__ zk, int N1, int B, int role, int g, bool store) {
  using K = KGC<N0>;
  constexpr int R1 = K::R1, HS = K::HS, G = K::G, RP = N0 / 2;
  const int kk = role == 0 ? 0 : N1;        // DC or Nyquist slot of the packed row spectra
  cp acc[R1];
#pragma unroll
  for (int s = 0; s < R1; ++s) acc[s] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  for (int b = 0; b < B; ++b) {
    float2 in[R1];
#pragma unroll
    for (int s = 0; s < HS; ++s) {
      const int rp = g + s * G;
      // packed rows (a + i b) hold real values at DC and Nyquist
      const float2 pu = zt_ld(zu + b * zvol + static_cast<long long>(kk) * RP + rp);
      const float2 pz = zt_ld(zz + b * zvol + static_cast<long long>(kk) * RP + rp);
      in[s] = make_float2(pu.x, pz.x);          // row a: u + i z
      in[s + HS] = make_float2(pu.y, pz.y);     // row b
    }
    cp x[R1], xp[R1];
    padded_fwd<N0>(in, x, g, buf, 0, t, 0u);
    fetch_partner<N0>(x, xp, g, buf, 0, 0u);
#pragma unroll
    for (int s = 0; s < R1; ++s) {
      // Im(W Wm) / 2 and -(|W|^2 - |Wm|^2) / 4 per path
      const float2 imww = pfma(x[s].re, xp[s].im, pmul(x[s].im, xp[s].re));
      const float2 nw = pfma(x[s].re, x[s].re, pmul(x[s].im, x[s].im));
      const float2 nwm = pfma(xp[s].re, xp[s].re, pmul(xp[s].im, xp[s].im));
      acc[s].re = pfma(f2(0.5f), imww, acc[s].re);
      acc[s].im = pfma(f2(-0.25f), psub(nw, nwm), acc[s].im);
    }
  }
  // A_DC + i A_Nyq on role 0
  cp a[R1];
#pragma unroll
  for (int s = 0; s < R1; ++s) {
    const cp n = shfl_cp(acc[s], G);
    a[s] = {psub(acc[s].re, n.im), padd(acc[s].im, n.re)};
  }
  float2 lo[R1], hi[R1];
  l1_full_inv<N0>(a, lo, hi, g, buf, t);
  if (store && role == 0) kg_column_out<N0>(zk, N1, 0, g, lo, hi);
}

// Wave layout: Zu, Zz [vol][2 n1][n0 / 2] (vol = channel-local cl B + b), Zk
// [cl][2 n1][n0] (row pairs (s0, s0 + n0) of the channel's offset grid).
// Column units cu = 1 .. n1 - 1 (blockIdx.x: channel, blockIdx.y: unit block).
template <int N0>
__global__ void __launch_bounds__(kTM, 2) k_kgcol(const float2* __restrict__ Zu, const float2* __restrict__ Zz,
                                               float2* __restrict__ Zk, int N1, int B) {
  using K = KGC<N0>;
  extern __shared__ __align__(16) unsigned char smem[];
  pdl_release();
  const Tabs<N0> t = tabs_at<N0>(smem);
  tabs_build<N0>(t, g_tw512);
  float4* xb = reinterpret_cast<float4*>(smem + Tabs<N0>::kBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pen = lane / K::G, g = lane % K::G;
  float4* buf = xb + warp * XB<N0>::kWarp + pen * XB<N0>::kPen;
  const int role = pen & 1;
  const int cu = 1 + blockIdx.y * K::UPB + warp * K::UPW + (pen >> 1);
  const int cl = blockIdx.x;
  const long long zvol = 2LL * N1 * (N0 / 2);
  const float2* zu = Zu + static_cast<long long>(cl) * B * zvol;
  const float2* zz = Zz + static_cast<long long>(cl) * B * zvol;
  float2* zk = Zk + static_cast<long long>(cl) * 2 * N1 * N0;
  __syncthreads();
  pdl_wait();
  kgcol_general<N0>(t, buf, zu, zz, zvol, zk, N1, B, cu, role, g);
}

// The combined DC/Nyquist unit of every channel of the wave: one warp per
// channel (blockIdx.x), pencils 0 and 1; further pencils of the warp run the
// same code without storing.
template <int N0>
__global__ void __launch_bounds__(32) k_kgcol_dc(const float2* __restrict__ Zu, const float2* __restrict__ Zz,
                                              float2* __restrict__ Zk, int N1, int B) {
  using K = KGC<N0>;
  extern __shared__ __align__(16) unsigned char smem[];
  pdl_release();
  const Tabs<N0> t = tabs_at<N0>(smem);
  tabs_build<N0>(t, g_tw512);
  float4* xb = reinterpret_cast<float4*>(smem + Tabs<N0>::kBytes);
  const int lane = threadIdx.x & 31;
  const int pen = lane / K::G, g = lane % K::G;
  float4* buf = xb + pen * XB<N0>::kPen;
  const int cl = blockIdx.x;
  const long long zvol = 2LL * N1 * (N0 / 2);
  __syncthreads();
  pdl_wait();
  kgcol_dc_nyquist<N0>(t, buf, Zu + static_cast<long long>(cl) * B * zvol, Zz + static_cast<long long>(cl) * B * zvol,
                       zvol, Zk + static_cast<long long>(cl) * 2 * N1 * N0, N1, B, pen & 1, g, (pen >> 1) == 0);
}

template <int N0>
struct KGCD {
  static constexpr size_t kBytes = Tabs<N0>::kBytes + 16ull * XB<N0>::kWarp;
};

// Inverse rows: the channel's packed row pairs (s0, s0 + n0), s0 in [0, n0),
// full-length inverse transform, read out at the offsets with the scale.
template <int NL>
__global__ void __launch_bounds__(kTM, 2) k_kginv(const float2* __restrict__ Zk, float* __restrict__ dK, int n0,
                                               int c0, float scale) {
  using R = RT<NL>;
  constexpr int G = R::G, PPW = R::PPW, R1 = P2<NL>::R1, RPB = R::RPB;
  static_assert(RPB == kWM * PPW, "one row pair per pencil");
  extern __shared__ __align__(16) unsigned char smem[];
  pdl_release();
  const Tabs<NL> t = tabs_at<NL>(smem);
  tabs_build<NL>(t, g_tw512);
  unsigned char* work = smem + Tabs<NL>::kBytes;
  float2* tile = reinterpret_cast<float2*>(work);
  float4* xb = reinterpret_cast<float4*>(work);
  const int cl = blockIdx.x, rpb = blockIdx.y * RPB;
  const float2* zk = Zk + static_cast<long long>(cl) * 2 * NL * n0;
  __syncthreads();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nrp = min(RPB, n0 - rpb);
  tile_from_ws<NL>(tile, zk, n0, rpb, nrp);
  task_sync();
  const int pen = lane / G, g = lane % G;
  const int rl = warp * PPW + pen;
  float4* buf = xb + warp * XB<NL>::kWarp + pen * XB<NL>::kPen;
  cp x[R1];
#pragma unroll
  for (int s = 0; s < R1; ++s) {
    const int kk = 2 * spec_idx<NL>(g, s);
    const float2 e = *HND_S(&tile[R::row(kk) + rl]), d = *HND_S(&tile[R::row(kk + 1) + rl]);
    x[s] = {make_float2(e.x, d.x), make_float2(e.y, d.y)};
  }
  task_sync();
  float2 lo[R1], hi[R1];
  l1_full_inv<NL>(x, lo, hi, g, buf, t);
  if (rl >= nrp) return;
  // rows s0 (real part, t0 = s0) and s0 + n0 (imaginary part, t0 = s0 - n0; none for s0 = 0);
  // columns s1 < n1 -> t1 = s1, s1 > n1 -> t1 = s1 - 2 n1 (slot n1 unused)
  const int s0 = rpb + rl;
  const long long W = 2LL * NL - 1;
  float* dkc = dK + static_cast<long long>(c0 + cl) * (2LL * n0 - 1) * W;
  float* ra = dkc + (static_cast<long long>(s0) + n0 - 1) * W;
  float* rb = dkc + (static_cast<long long>(s0) - 1) * W;
#pragma unroll
  for (int s = 0; s < R1; ++s) {
    const int s1 = g + s * G;
    // lo: column s1 (t1 = s1, index s1 + n1 - 1); hi: column s1 + n1 (t1 = s1 - n1, index s1 - 1; none for s1 = 0)
    *HND_G(&ra[s1 + NL - 1]) = lo[s].x * scale;
    if (s1 > 0) *HND_G(&ra[s1 - 1]) = hi[s].x * scale;
    if (s0 > 0) {
      *HND_G(&rb[s1 + NL - 1]) = lo[s].y * scale;
      if (s1 > 0) *HND_G(&rb[s1 - 1]) = hi[s].y * scale;
    }
  }
}

}  // namespace hnd2
