// hnd_multi2.cuh -- multi-pass tiers on the packed two-path FFT core, for
// volumes whose padded transform does not fit one SM (2D with an axis >= 128,
// every 3D grid).  One wave of (b, c) volumes at a time:
//   k_rowfwd2   rows along the last axis, packed two at a time, zero-padded
//               forward transform -> Zt[kk][rp] (an L2-sized workspace)
//   k_mid1v2    2D: per last-axis frequency, zero-padded convolution along
//               axis 0 with the channel spectrum
//   k_mid2v2    3D: per last-axis frequency, zero-padded 2D convolution over
//               axes (0, 1)
//   k_rowinv2   inverse rows, crop, output gate q
// (HyenaND pages: zero padding to twice the grid; forward FFT, spectral
// modulation, inverse FFT and output cropping.)
#pragma once

#include "hnd_fused2.cuh"

#include <cooperative_groups.h>

namespace hnd2 {

namespace cg = cooperative_groups;

constexpr int kTM = 256;          // threads per CTA in the multi-pass kernels

constexpr int kWM = kTM / 32;

// Barrier over the kTM task threads (named barrier 1).  In the stage kernels
// these are all the threads of the CTA; the persistent pipeline adds a
// scheduler warp that does not take part.
__device__ __forceinline__ void task_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kTM) : "memory"); }


// ------------------------------------------------------ workspace access
// The wave workspace (packed row spectra) bypasses L1: it is written by one
// stage kernel and read by the next.  (An L2 evict-last policy on these
// accesses, to keep a wave resident while the activations stream past, was
// measured 2% slower on the 256^2 grid and is not used.)
__device__ __forceinline__ float2 zt_ld(const float2* p) { return __ldcg(HND_G(p)); }
__device__ __forceinline__ float4 zt_ld(const float4* p) { return __ldcg(HND_G(p)); }
__device__ __forceinline__ void zt_st(float2* p, float2 v) { __stcg(HND_G(p), v); }
__device__ __forceinline__ void zt_st(float4* p, float4 v) { __stcg(HND_G(p), v); }

// Row pair rp = rows (ra, ra + ps): 2D pairs row r with r + n0/2 (ps = n0/2),
// 3D pairs neighbouring rows (ps = 1).
__device__ __forceinline__ long long pair_row(long long rp, int ps) { return (rp / ps) * 2 * ps + (rp % ps); }

// Row tile: for each of the 2 NL frequencies kk, RPB row pairs (float2).
// Even and odd frequencies sit in two planes, row f = kk / 2 at f TS of its
// plane.  A pencil's lanes hold consecutive f, so with the pitch TS = 16 / G
// (mod 16) the lanes and pencils of a half-warp hit 16 distinct 8-byte bank
// slots when they write or gather a frequency row; an even pitch keeps rows
// 16-byte aligned for the workspace-side float4 accesses, and for the odd
// pitch (G = 16) the odd plane is shifted by one slot so that the two planes'
// rows read by one half-warp interleave.
template <int NL>
struct RT {
  static constexpr int G = P2<NL>::G, PPW = 32 / G;
  static constexpr int RPB = (kWM * PPW) * ((kWM * PPW) < 16 ? 2 : 1);   // row pairs per CTA
  static constexpr int TS = RPB + ((16 / G - RPB) % 16 + 16) % 16;       // tile pitch (float2)
  static constexpr int PL = NL * TS + TS % 2;                            // plane stride (float2)
  // The row tile and the FFT exchange buffers are never live together, so
  // they share one region.
  static constexpr size_t kTile = sizeof(float2) * 2 * PL;
  static constexpr size_t kXb = 16ull * XB<NL>::kWarp * kWM;
  static constexpr size_t kBytes = Tabs<NL>::kBytes + (kTile > kXb ? kTile : kXb);
  static __device__ __forceinline__ int row(int kk) { return (kk & 1) * PL + (kk >> 1) * TS; }
};

// Tile <-> workspace copies: rows of RPB row pairs (float2) per frequency kk,
// moved as float4 pairs, every load of a thread issued before its stores.
template <int NL>
__device__ __forceinline__ void tile_from_ws(float2* tile, const float2* __restrict__ zt, int rp_total, int rpb,
                                             int nrp) {
  using R = RT<NL>;
  constexpr int RPB = R::RPB;
  constexpr int PER = NL * RPB / kTM;                     // float4 per thread
  static_assert(PER * kTM == NL * RPB && RPB % 2 == 0, "tile split");
  float4 v[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = 2 * (threadIdx.x + i * kTM);
    const int kk = e / RPB, rl = e % RPB;
    const float2* src = zt + static_cast<long long>(kk) * rp_total + rpb + rl;
    if (rl + 1 < nrp) {
      v[i] = zt_ld(reinterpret_cast<const float4*>(src));
    } else {
      const float2 a = rl < nrp ? zt_ld(src) : make_float2(0.f, 0.f);
      v[i] = make_float4(a.x, a.y, 0.f, 0.f);
    }
  }
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = 2 * (threadIdx.x + i * kTM);
    const int kk = e / RPB, rl = e % RPB;
    float2* t = tile + R::row(kk) + rl;
    if constexpr (R::TS % 2 == 0) {
      *HND_S(reinterpret_cast<float4*>(t)) = v[i];
    } else {
      *HND_S(&t[0]) = make_float2(v[i].x, v[i].y);
      *HND_S(&t[1]) = make_float2(v[i].z, v[i].w);
    }
  }
}

template <int NL>
__device__ __forceinline__ void tile_to_ws(const float2* tile, float2* __restrict__ zt, int rp_total, int rpb,
                                           int nrp) {
  using R = RT<NL>;
  constexpr int RPB = R::RPB;
  constexpr int PER = NL * RPB / kTM;
  static_assert(PER * kTM == NL * RPB && RPB % 2 == 0, "tile split");
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = 2 * (threadIdx.x + i * kTM);
    const int kk = e / RPB, rl = e % RPB;
    const float2* t = tile + R::row(kk) + rl;
    float2 a, b;
    if constexpr (R::TS % 2 == 0) {
      const float4 ab = *HND_S(reinterpret_cast<const float4*>(t));
      a = make_float2(ab.x, ab.y), b = make_float2(ab.z, ab.w);
    } else {
      a = *HND_S(&t[0]), b = *HND_S(&t[1]);
    }
    float2* dst = zt + static_cast<long long>(kk) * rp_total + rpb + rl;
    if (rl + 1 < nrp) {
      zt_st(reinterpret_cast<float4*>(dst), make_float4(a.x, a.y, b.x, b.y));
    } else if (rl < nrp) {
      zt_st(dst, a);
    }
  }
}

// ------------------------------------------------------------- forward rows
// One task: RPB row pairs starting at rpb of one volume (activations at
// `base`, workspace `ztv`).  `work` is the shared region after the tables.
template <int NL, class T>
__device__ __forceinline__ void rowfwd_task(const Tabs<NL> t, unsigned char* work, const T* __restrict__ k,
                                            const T* __restrict__ v, float2* __restrict__ ztv, long long base,
                                            int rpb, int rp_total, int ps) {
  using R = RT<NL>;
  constexpr int G = R::G, PPW = R::PPW, R1 = P2<NL>::R1, RPB = R::RPB;
  float2* tile = reinterpret_cast<float2*>(work);
  float4* xb = reinterpret_cast<float4*>(work);     // shares the tile region
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nrp = min(RPB, rp_total - rpb);
  const int pen = lane / G, g = lane % G;
  float4* buf = xb + warp * XB<NL>::kWarp + pen * XB<NL>::kPen;
  static_assert(RPB == kWM * PPW || RPB == 2 * kWM * PPW, "row tile covers one or two rounds");
  constexpr int ROUNDS = RPB / (kWM * PPW);
  cp keep[ROUNDS > 1 ? R1 : 1];
  for (int round = 0; round < ROUNDS; ++round) {
    const int r0 = round * kWM * PPW + warp * PPW;
    const int rl = r0 + pen;
    const bool act = rl < nrp;
    const long long ra = pair_row(rpb + rl, ps) * NL, rb = ra + static_cast<long long>(ps) * NL;
    float2 z[R1];
#pragma unroll
    for (int s = 0; s < R1; ++s) {
      const long long j = g + s * G;
      z[s] = act ? make_float2(Act<T>::ld_g(k + base + ra + j) * Act<T>::ld_g(v + base + ra + j),
                               Act<T>::ld_g(k + base + rb + j) * Act<T>::ld_g(v + base + rb + j))
                 : make_float2(0.f, 0.f);
    }
    cp x[R1];
    padded_fwd<NL>(z, x, g, buf, 0, t, 0u);
    if (ROUNDS > 1 && round == 0) {
#pragma unroll
      for (int s = 0; s < R1; ++s) keep[ROUNDS > 1 ? s : 0] = x[s];
      continue;
    }
    task_sync();      // every pencil's exchange buffer is free: reuse it as the tile
    auto put = [&](const cp (&xx)[R1], int rl_) {
#pragma unroll
      for (int s = 0; s < R1; ++s) {
        const int kk = 2 * spec_idx<NL>(g, s);
        *HND_S(&tile[R::row(kk) + rl_]) = make_float2(xx[s].re.x, xx[s].im.x);
        *HND_S(&tile[R::row(kk + 1) + rl_]) = make_float2(xx[s].re.y, xx[s].im.y);
      }
    };
    if constexpr (ROUNDS > 1) put(keep, warp * PPW + pen);
    put(x, rl);
  }
  task_sync();
  tile_to_ws<NL>(tile, ztv, rp_total, rpb, nrp);
}

template <int NL, class T>
__global__ void __launch_bounds__(kTM, 2) k_rowfwd2(const T* __restrict__ k, const T* __restrict__ v,
                                                 float2* __restrict__ Zt, long long ord0, int rp_total, int ps,
                                                 int B, int C) {
  extern __shared__ __align__(16) unsigned char smem[];
  pdl_release();
  const Tabs<NL> t = tabs_at<NL>(smem);
  tabs_build<NL>(t, g_tw512);
  const long long ord = ord0 + blockIdx.x;
  const int c = static_cast<int>(ord / B), b = static_cast<int>(ord % B);
  const long long L = static_cast<long long>(rp_total) * 2 * NL;
  __syncthreads();
  pdl_wait();
  rowfwd_task<NL, T>(t, smem + Tabs<NL>::kBytes, k, v, Zt + static_cast<long long>(blockIdx.x) * L,
                     (static_cast<long long>(b) * C + c) * L, blockIdx.y * RT<NL>::RPB, rp_total, ps);
}

// ------------------------------------------------------------- inverse rows
template <int NL, class T>
__device__ __forceinline__ void rowinv_task(const Tabs<NL> t, unsigned char* work, const float2* __restrict__ ztv,
                                            const T* __restrict__ q, T* __restrict__ y, long long base, int rpb,
                                            int rp_total, int ps, const T* __restrict__ g2 = nullptr,
                                            T* __restrict__ y2 = nullptr) {
  using R = RT<NL>;
  constexpr int G = R::G, PPW = R::PPW, R1 = P2<NL>::R1, RPB = R::RPB;
  float2* tile = reinterpret_cast<float2*>(work);
  float4* xb = reinterpret_cast<float4*>(work);     // shares the tile region
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nrp = min(RPB, rp_total - rpb);
  const int pen = lane / G, g = lane % G;
  float4* buf = xb + warp * XB<NL>::kWarp + pen * XB<NL>::kPen;
  static_assert(RPB == kWM * PPW || RPB == 2 * kWM * PPW, "row tile covers one or two rounds");
  constexpr int ROUNDS = RPB / (kWM * PPW);
  cp xin[ROUNDS][R1];
  {
    tile_from_ws<NL>(tile, ztv, rp_total, rpb, nrp);
    task_sync();
    // pull every round's inputs out of the tile before the tile region turns
    // into exchange buffers
#pragma unroll
    for (int round = 0; round < ROUNDS; ++round) {
      const int rl = round * kWM * PPW + warp * PPW + pen;
#pragma unroll
      for (int s = 0; s < R1; ++s) {
        const int kk = 2 * spec_idx<NL>(g, s);
        const float2 e = *HND_S(&tile[R::row(kk) + rl]), d = *HND_S(&tile[R::row(kk + 1) + rl]);
        xin[round][s] = {make_float2(e.x, d.x), make_float2(e.y, d.y)};
      }
    }
    task_sync();
  }
  for (int round = 0; round < ROUNDS; ++round) {
    const int r0 = round * kWM * PPW + warp * PPW;
    const int rl = r0 + pen;
    const bool act = rl < nrp;
    const long long ra = pair_row(rpb + rl, ps) * NL, rb = ra + static_cast<long long>(ps) * NL;
    float qa[R1], qb[R1];
#pragma unroll
    for (int s = 0; s < R1; ++s) {
      const long long j = g + s * G;
      qa[s] = act ? Act<T>::ld_g(q + base + ra + j) : 0.f;
      qb[s] = act ? Act<T>::ld_g(q + base + rb + j) : 0.f;
    }
    cp x[R1];
#pragma unroll
    for (int s = 0; s < R1; ++s) x[s] = xin[round][s];
    float2 o[R1];
    padded_inv<NL>(x, o, g, buf, 0, t, 0u);
    if (act) {
#pragma unroll
      for (int s = 0; s < R1; ++s) {
        const long long j = g + s * G;
        Act<T>::st_g(y + base + ra + j, o[s].x * qa[s]);
        Act<T>::st_g(y + base + rb + j, o[s].y * qb[s]);
      }
      if (y2) {       // second gated output of the same convolution
#pragma unroll
        for (int s = 0; s < R1; ++s) {
          const long long j = g + s * G;
          Act<T>::st_g(y2 + base + ra + j, o[s].x * Act<T>::ld_g(g2 + base + ra + j));
          Act<T>::st_g(y2 + base + rb + j, o[s].y * Act<T>::ld_g(g2 + base + rb + j));
        }
      }
    }
  }
}

template <int NL, class T>
__global__ void __launch_bounds__(kTM, 2) k_rowinv2(const float2* __restrict__ Zt, const T* __restrict__ q,
                                                 T* __restrict__ y, long long ord0, int rp_total, int ps, int B,
                                                 int C, const T* __restrict__ g2, T* __restrict__ y2) {
  extern __shared__ __align__(16) unsigned char smem[];
  pdl_release();
  const Tabs<NL> t = tabs_at<NL>(smem);
  tabs_build<NL>(t, g_tw512);
  const long long ord = ord0 + blockIdx.x;
  const int c = static_cast<int>(ord / B), b = static_cast<int>(ord % B);
  const long long L = static_cast<long long>(rp_total) * 2 * NL;
  __syncthreads();
  pdl_wait();
  rowinv_task<NL, T>(t, smem + Tabs<NL>::kBytes, Zt + static_cast<long long>(blockIdx.x) * L, q, y,
                     (static_cast<long long>(b) * C + c) * L, blockIdx.y * RT<NL>::RPB, rp_total, ps, g2, y2);
}

// ---------------------------------------------------------- 2D column units
// Zt[kk][rp] per volume, rp in [0, n0/2) with row pair (rp, rp + n0/2); unit cu
// = last-axis frequency kx (cu >= 1) or the combined DC/Nyquist unit (cu = 0).
template <int N0>
struct M1 {
  static constexpr int G = P2<N0>::G, PPW = 32 / G;
  static constexpr int UPB = kWM * PPW;                  // units per CTA
  static constexpr size_t kBytes = Tabs<N0>::kBytes + 16ull * XB<N0>::kWarp * kWM;
};

#ifndef HND_MID1_PREFETCH
#define HND_MID1_PREFETCH 1
#endif

// One column unit cu (one pencil of lanes).  GEN: the warp that holds unit
// 0, the combined DC/Nyquist unit, whose product needs the partner
// frequency; every pencil of that warp takes this path (for cu != 0 the
// partner term is multiplied by zero).
template <int N0, bool GEN, bool CONJ>
__device__ __forceinline__ void mid1_unit(const Tabs<N0> t, float4* buf, float2* __restrict__ zt,
                                          const float4* __restrict__ sp, int N1, int cu, int g) {
  constexpr float sgn = CONJ ? -1.f : 1.f;      // -1: conjugate spectrum (the adjoint)
  constexpr int G = P2<N0>::G, R1 = P2<N0>::R1, RP = N0 / 2, HS = R1 / 2;
  const bool act = cu < N1;
  const int kx = act ? cu : 1, kxm = cu == 0 ? N1 : 2 * N1 - kx;
  float2 z[R1];
#pragma unroll
  for (int s = 0; s < HS; ++s) {
    const int rp = g + s * G;
    float2 z1 = make_float2(0.f, 0.f), z2 = z1;
    if (act) {
      z1 = zt_ld(zt + static_cast<long long>(kx) * RP + rp);
      z2 = zt_ld(zt + static_cast<long long>(kxm) * RP + rp);
    }
    if (cu == 0) {
      z[s] = make_float2(z1.x, z2.x);
      z[s + HS] = make_float2(z1.y, z2.y);
    } else {
      z[s] = unpack_a(z1, z2);
      z[s + HS] = unpack_b(z1, z2);
    }
  }
  const float4* su = sp + (cu == 0 ? 0LL : static_cast<long long>(cu + 1) * N0);
#if HND_MID1_PREFETCH
  // the unit's spectrum comes from HBM: start fetching it before the forward
  // transform so that the product after it does not wait the full latency
  if (act) {
#pragma unroll
    for (int s = 0; s < R1; ++s) {
#if HND_MID1_PREFETCH == 2
      if (HND_RANGE_OK(su + s * G + g, 16)) asm volatile("prefetch.global.L1 [%0];" ::"l"(su + s * G + g));
#else
      if (HND_RANGE_OK(su + s * G + g, 16)) asm volatile("prefetch.global.L2 [%0];" ::"l"(su + s * G + g));
#endif
    }
  }
#endif
  cp x[R1];
  padded_fwd<N0>(z, x, g, buf, 0, t, 0u);
  if constexpr (GEN) {
    cp xp[R1];
    fetch_partner<N0>(x, xp, g, buf, 0, 0u);
#pragma unroll
    for (int s = 0; s < R1; ++s) {
      float4 S = act ? __ldg(HND_G(su + s * G + g)) : make_float4(0.f, 0.f, 0.f, 0.f);
      float4 Bc = (cu == 0) ? __ldg(HND_G(sp + N0 + s * G + g)) : make_float4(0.f, 0.f, 0.f, 0.f);
      S.z *= sgn, S.w *= sgn, Bc.z *= sgn, Bc.w *= sgn;     // sgn = -1: conjugate spectrum (adjoint)
      const cp a = cmulp(x[s], make_float2(S.x, S.y), make_float2(S.z, S.w));
      const cp xc = {xp[s].re, make_float2(-xp[s].im.x, -xp[s].im.y)};
      const cp bb = cmulp(xc, make_float2(Bc.x, Bc.y), make_float2(Bc.z, Bc.w));
      x[s] = cadd(a, bb);
    }
  } else {
    if (act) {
#pragma unroll
      for (int s = 0; s < R1; ++s) {
        const float4 S = __ldg(HND_G(su + s * G + g));
        x[s] = cmulp(x[s], make_float2(S.x, S.y), make_float2(sgn * S.z, sgn * S.w));
      }
    }
  }
  float2 o[R1];
  padded_inv<N0>(x, o, g, buf, 0, t, 0u);
  if (act) {
#pragma unroll
    for (int s = 0; s < HS; ++s) {
      const int rp = g + s * G;
      const float2 ya = o[s], yb = o[s + HS];
      if (cu == 0) {
        zt_st(zt + rp, make_float2(ya.x, yb.x));
        zt_st(zt + static_cast<long long>(N1) * RP + rp, make_float2(ya.y, yb.y));
      } else {
        zt_st(zt + static_cast<long long>(kx) * RP + rp, pack_pos(ya, yb));
        zt_st(zt + static_cast<long long>(kxm) * RP + rp, pack_neg(ya, yb));
      }
    }
  }
}

// The DC/Nyquist warp's path, kept out of line so that its extra registers
// do not weigh on the common path.  (The checked build, with relocatable
// device code, keeps it inline: an out-of-line function there gets its own
// register budget, above the kernel's.)
#ifdef HYENA_ND_BOUNDS
#define HND_OUT_OF_LINE __forceinline__
#else
#define HND_OUT_OF_LINE __noinline__
#endif
template <int N0, bool CONJ>
__device__ HND_OUT_OF_LINE void mid1_unit_gen(const Tabs<N0> t, float4* buf, float2* __restrict__ zt,
                                           const float4* __restrict__ sp, int N1, int cu, int g) {
  mid1_unit<N0, true, CONJ>(t, buf, zt, sp, N1, cu, g);
}

// One task: UPB column units starting at u0 of one volume; `sp` is the
// channel's spectrum for this sample.
template <int N0, bool CONJ>
__device__ __forceinline__ void mid1_task(const Tabs<N0> t, unsigned char* work, float2* __restrict__ zt,
                                          const float4* __restrict__ sp, int N1, int u0) {
  using M = M1<N0>;
  constexpr int G = M::G, PPW = M::PPW;
  float4* xb = reinterpret_cast<float4*>(work);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pen = lane / G, g = lane % G;
  float4* buf = xb + warp * XB<N0>::kWarp + pen * XB<N0>::kPen;
  const int cu = u0 + warp * PPW + pen;
  if (u0 == 0 && warp == 0) mid1_unit_gen<N0, CONJ>(t, buf, zt, sp, N1, cu, g);
  else mid1_unit<N0, false, CONJ>(t, buf, zt, sp, N1, cu, g);
}

template <int N0, bool CONJ>
__global__ void __launch_bounds__(kTM, 2) k_mid1v2(float2* __restrict__ Zt, const float4* __restrict__ spec,
                                                long long sbs4, int N1, long long ord0, int B, int C) {
  extern __shared__ __align__(16) unsigned char smem[];
  pdl_release();
  const Tabs<N0> t = tabs_at<N0>(smem);
  tabs_build<N0>(t, g_tw512);
  const long long ord = ord0 + blockIdx.x;
  const int c = static_cast<int>(ord / B), b = static_cast<int>(ord % B);
  const float4* sp = spec + static_cast<long long>(b) * sbs4 + static_cast<long long>(c) * (N1 + 1) * N0;
  __syncthreads();
  pdl_wait();
  mid1_task<N0, CONJ>(t, smem + Tabs<N0>::kBytes, Zt + static_cast<long long>(blockIdx.x) * 2 * N1 * (N0 / 2), sp, N1,
                blockIdx.y * M1<N0>::UPB);
}

// ---------------------------------------------------------------- 3D slabs
// For one last-axis frequency kx: the (axis 0, axis 1) slab of both packed
// rows' spectra (rows y and y + 1 share one Zt entry), zero-padded 2D
// convolution with the channel's slab spectrum, written back packed.
//   step 1  y transforms (one pencil per z)       -> F[ky][z]
//   step 2  z-pencil convolution per ky (spectrum payload [s][g] per ky)
//   step 3  inverse y transforms, repack, write Zt
// With HALF = true the slab is split over a 2-CTA cluster by ky parity: CTA h
// keeps ky = 2m + h and finishes rows z in [h n0/2, (h + 1) n0/2), reading the
// other parity through distributed shared memory.
template <int N0, int N1, bool HALF>
struct M2 {
  static constexpr int FS = N0 + 1;
  static constexpr int NKY = HALF ? N1 : 2 * N1;         // ky rows held by this CTA
  static constexpr size_t kTabs = Tabs<N0>::kBytes + (N0 == N1 ? 0 : Tabs<N1>::kBytes);
  static constexpr int XW = XB<N0>::kWarp > XB<N1>::kWarp ? XB<N0>::kWarp : XB<N1>::kWarp;
  static constexpr size_t kBytes = kTabs + sizeof(float2) * NKY * FS + 16ull * XW * kWM;
};

template <int N0, int N1>
__device__ __forceinline__ void slab_rows_in(const float2* __restrict__ zt, long long RPn, int kx, int kxm,
                                            bool self_conj, int z, int g, float2 (&x)[P2<N1>::R1]) {
  constexpr int G = P2<N1>::G, R1 = P2<N1>::R1;
#pragma unroll
  for (int s = 0; s < R1; ++s) {
    const int yy = g + s * G;
    const long long rp = (static_cast<long long>(z) * N1 + yy) >> 1;
    const float2 z1 = zt_ld(zt + kx * RPn + rp);
    const float2 z2 = self_conj ? z1 : zt_ld(zt + kxm * RPn + rp);
    x[s] = (yy & 1) ? unpack_b(z1, z2) : unpack_a(z1, z2);
  }
}

template <int N0, int N1>
__device__ __forceinline__ void slab_rows_out(float2* __restrict__ zt, long long RPn, int kx, int kxm, bool self_conj,
                                             int z, int g, bool act, const float2 (&o)[P2<N1>::R1]) {
  constexpr int G = P2<N1>::G, R1 = P2<N1>::R1;
#pragma unroll
  for (int s = 0; s < R1; ++s) {
    const float2 own = o[s];
    float2 oth;
    if constexpr (G >= 2) {
      oth.x = __shfl_xor_sync(0xffffffffu, own.x, 1);
      oth.y = __shfl_xor_sync(0xffffffffu, own.y, 1);
    } else {
      oth = o[s ^ 1];
    }
    const int yy = g + s * G;
    const long long rp = (static_cast<long long>(z) * N1 + yy) >> 1;
    const bool odd = yy & 1;
    const float2 ya = odd ? oth : own, yb = odd ? own : oth;
    if (!act) continue;
    if (self_conj) {
      if (!odd) zt_st(zt + kx * RPn + rp, make_float2(ya.x, yb.x));
    } else {
      if (!odd) zt_st(zt + kx * RPn + rp, pack_pos(ya, yb));
      else zt_st(zt + kxm * RPn + rp, pack_neg(ya, yb));
    }
  }
}

// One task: the slab of last-axis frequency kx of one volume (`zt`), with the
// channel's slab spectrum `sslab` for this sample.  `work` holds F, then the
// exchange buffers.
template <int N0, int N1, bool HALF, bool CONJ>
__device__ __forceinline__ void mid2_task(const Tabs<N0> t0, const Tabs<N1> t1, unsigned char* work,
                                          float2* __restrict__ zt, const float4* __restrict__ sslab, int N2, int kx,
                                          int h) {
  constexpr float sgn = CONJ ? -1.f : 1.f;      // -1: conjugate spectrum (the adjoint)
  using M = M2<N0, N1, HALF>;
  constexpr int FS = M::FS, NKY = M::NKY;
  constexpr int G0 = P2<N0>::G, R0 = P2<N0>::R1, G1 = P2<N1>::G, R1 = P2<N1>::R1;
  float2* F = reinterpret_cast<float2*>(work);
  float4* xb = reinterpret_cast<float4*>(work + sizeof(float2) * NKY * FS);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long RPn = static_cast<long long>(N0) * N1 / 2;
  const bool self_conj = (kx == 0) || (kx == N2);
  const int kxm = self_conj ? kx : 2 * N2 - kx;
  // step 1: y transforms, one pencil per z
  {
    constexpr int PPW = 32 / G1;
    const int pen = lane / G1, g = lane % G1;
    float4* buf = xb + warp * M::XW + pen * XB<N1>::kPen;
    for (int z0 = warp * PPW; z0 < N0; z0 += kWM * PPW) {
      const int z = z0 + pen;
      const bool act = z < N0;
      float2 in[R1];
      if (act) {
        slab_rows_in<N0, N1>(zt, RPn, kx, kxm, self_conj, z, g, in);
      } else {
#pragma unroll
        for (int s = 0; s < R1; ++s) in[s] = make_float2(0.f, 0.f);
      }
      cp x[R1];
      padded_fwd<N1>(in, x, g, buf, 0, t1, 0u);
      if (act) {
#pragma unroll
        for (int s = 0; s < R1; ++s) {
          const int f = spec_idx<N1>(g, s);
          if (HALF) {
            *HND_S(&F[f * FS + z]) = h == 0 ? make_float2(x[s].re.x, x[s].im.x) : make_float2(x[s].re.y, x[s].im.y);
          } else {
            *HND_S(&F[(2 * f) * FS + z]) = make_float2(x[s].re.x, x[s].im.x);
            *HND_S(&F[(2 * f + 1) * FS + z]) = make_float2(x[s].re.y, x[s].im.y);
          }
        }
      }
    }
  }
  task_sync();
  // step 2: z-pencil convolution per ky row held here; pencils of a warp
  // take rows 8 apart (bank groups of F)
  {
    constexpr int PPW = 32 / G0, SLOTS = kWM * PPW;
    const int pen = lane / G0, g = lane % G0;
    float4* buf = xb + warp * XB<N0>::kWarp + pen * XB<N0>::kPen;
    for (int r0 = 0; r0 < NKY; r0 += SLOTS) {
      const int kyl = r0 + warp + pen * kWM;
      const bool act = kyl < NKY;
      const int ky = HALF ? 2 * kyl + h : kyl;
      const float4* su = sslab + static_cast<long long>(act ? ky : 0) * N0;
      constexpr int NPF = R0 == 8 ? 8 : 1;             // prefetch the payload when registers allow
      float4 S[NPF];
      if (R0 == 8 && act) {
#pragma unroll
        for (int s = 0; s < NPF; ++s) S[s] = __ldg(HND_G(su + s * G0 + g));
      }
      float2 in[R0];
#pragma unroll
      for (int s = 0; s < R0; ++s) in[s] = act ? *HND_S(&F[kyl * FS + g + s * G0]) : make_float2(0.f, 0.f);
      cp x[R0];
      padded_fwd<N0>(in, x, g, buf, 0, t0, 0u);
      if (act) {
#pragma unroll
        for (int s = 0; s < R0; ++s) {
          const float4 Sv = (R0 == 8) ? S[s % NPF] : __ldg(HND_G(su + s * G0 + g));
          x[s] = cmulp(x[s], make_float2(Sv.x, Sv.y), make_float2(sgn * Sv.z, sgn * Sv.w));
        }
      }
      float2 o[R0];
      padded_inv<N0>(x, o, g, buf, 0, t0, 0u);
      if (act) {
#pragma unroll
        for (int s = 0; s < R0; ++s) *HND_S(&F[kyl * FS + g + s * G0]) = o[s];
      }
    }
  }
  if constexpr (HALF) {
    cg::this_cluster().sync();
  } else {
    task_sync();
  }
  // step 3: inverse y transforms, repack, write back
  {
    constexpr int PPW = 32 / G1;
    const int pen = lane / G1, g = lane % G1;
    float4* buf = xb + warp * M::XW + pen * XB<N1>::kPen;
    const float2* Fe = F;
    const float2* Fo = F;
    if constexpr (HALF) {
      float2* other = cg::this_cluster().map_shared_rank(F, h ^ 1);
      Fe = h == 0 ? F : other;
      Fo = h == 0 ? other : F;
    }
    constexpr int NZ = HALF ? N0 / 2 : N0;
    for (int z0 = warp * PPW; z0 < NZ; z0 += kWM * PPW) {
      const int zl = z0 + pen;
      const bool act = zl < NZ;
      const int z = HALF ? h * (N0 / 2) + zl : zl;
      cp x[R1];
#pragma unroll
      for (int s = 0; s < R1; ++s) {
        const int f = spec_idx<N1>(g, s);
        float2 e = make_float2(0.f, 0.f), d = e;
        if (act) {
          if (HALF) {
            if (HND_RANGE_OK(&F[f * FS + z], sizeof(float2))) {
              e = Fe[f * FS + z];
              d = Fo[f * FS + z];
            }
          } else {
            e = *HND_S(&F[(2 * f) * FS + z]);
            d = *HND_S(&F[(2 * f + 1) * FS + z]);
          }
        }
        x[s] = {make_float2(e.x, d.x), make_float2(e.y, d.y)};
      }
      float2 o[R1];
      padded_inv<N1>(x, o, g, buf, 0, t1, 0u);
      slab_rows_out<N0, N1>(zt, RPn, kx, kxm, self_conj, z, g, act, o);
    }
  }
  if constexpr (HALF) cg::this_cluster().sync();
}

template <int N0, int N1, bool HALF, bool CONJ>
__device__ __forceinline__ void mid2_kernel_body(float2* __restrict__ Zt, const float4* __restrict__ spec,
                                                 long long sbs4, int N2, long long ord0, int B, int C, int vol_local,
                                                 int h) {
  using M = M2<N0, N1, HALF>;
  extern __shared__ __align__(16) unsigned char smem[];
  pdl_release();
  const Tabs<N0> t0 = tabs_at<N0>(smem);
  Tabs<N1> t1;
  if constexpr (N0 == N1) {
    t1 = t0;
  } else {
    t1 = tabs_at<N1>(smem + Tabs<N0>::kBytes);
  }
  tabs_build<N0>(t0, g_tw512);
  if constexpr (N0 != N1) tabs_build<N1>(t1, g_tw512);
  const long long ord = ord0 + vol_local;
  const int c = static_cast<int>(ord / B), b = static_cast<int>(ord % B);
  const long long RPn = static_cast<long long>(N0) * N1 / 2;
  const int kx = blockIdx.y;
  const long long slab = 2LL * N1 * N0;                 // float4 per slab
  const float4* sslab = spec + static_cast<long long>(b) * sbs4 + static_cast<long long>(c) * (N2 + 1) * slab +
                        static_cast<long long>(kx) * slab;
  __syncthreads();
  pdl_wait();
  mid2_task<N0, N1, HALF, CONJ>(t0, t1, smem + M::kTabs, Zt + static_cast<long long>(vol_local) * 2 * N2 * RPn, sslab,
                                N2, kx, h);
}

template <int N0, int N1, bool CONJ>
__global__ void __launch_bounds__(kTM, 2) k_mid2v2(float2* __restrict__ Zt, const float4* __restrict__ spec,
                                                long long sbs4, int N2, long long ord0, int B, int C) {
  mid2_kernel_body<N0, N1, false, CONJ>(Zt, spec, sbs4, N2, ord0, B, C, blockIdx.x, 0);
}

template <int N0, int N1, bool CONJ>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kTM)
    k_mid2v2_pair(float2* __restrict__ Zt, const float4* __restrict__ spec, long long sbs4, int N2, long long ord0,
                  int B, int C) {
  const int h = static_cast<int>(cg::this_cluster().block_rank());
  mid2_kernel_body<N0, N1, true, CONJ>(Zt, spec, sbs4, N2, ord0, B, C, blockIdx.x / 2, h);
}

// --------------------------------------------------- spectrum layouts (v2)
// 3D, per channel, float4 units: for kx in [0, n2], for ky in [0, 2 n1), n0
// float4 at [s][g] of the z-pencil plan: (S[2f].re, S[2f+1].re, S[2f].im,
// S[2f+1].im), f = spec_idx(g, s), the z frequency of lane g, slot s.
__host__ __device__ __forceinline__ int spec_idx_gen(int N, int g, int s) {
  if (N == 8) return s;
  const int R1 = N >= 128 ? 16 : 8, R2 = N / R1, G = R2;
  return g + G * (s / R2) + (s % R2) * R1;
}
__host__ __device__ __forceinline__ int lanes_of(int N) { return N == 8 ? 1 : N / (N >= 128 ? 16 : 8); }

// natural half spectrum [C][2n0][2n1][n2 + 1] (pitch = last-axis length of the
// source: n2 + 1 for a half spectrum, 2 n2 for a full grid; pair: the filter
// call's full grids, two channels per grid) -> library order.
// A CTA takes one ky and kS3 consecutive kx of one source grid: it reads the
// z-pencils of those kx into shared memory (kx adjacent in the source, so a
// kz row is one contiguous read) and, for a pair grid, the z-pencils of the
// mirrored frequencies (-ky, -kx), again contiguous runs; it then writes the
// library's n0 float4 of each kx in slot order, contiguous -- for a pair grid
// both channels from the same reads (S_c = (W + conj W_m)/2,
// S_{c+1} = (W - conj W_m)/(2i)).
constexpr int kS3 = 16;
__host__ __device__ __forceinline__ size_t spec3_in_smem(int n0) { return sizeof(float2) * 2 * (2 * n0) * (kS3 + 1); }

static __global__ void __launch_bounds__(256) k_spec3_in(const float2* __restrict__ nat, float4* __restrict__ out,
                                                         int n0, int n1, int n2, long long C, long long pitch,
                                                         float scale, int pair = 0) {
  extern __shared__ __align__(16) float2 tw[];     // W [kz][kS3 + 1], then W_m [kz][kS3 + 1]
  float2* tm = tw + 2 * n0 * (kS3 + 1);
  const long long src_per = 4LL * n0 * n1 * pitch;
  const int nkb = (n2 + 1 + kS3 - 1) / kS3;
  const long long cta = blockIdx.x;
  const int kb0 = static_cast<int>(cta % nkb) * kS3;
  const int ky = static_cast<int>((cta / nkb) % (2 * n1));
  const long long gi = cta / (static_cast<long long>(nkb) * 2 * n1);   // source grid (pair) or channel
  const int nk = min(kS3, n2 + 1 - kb0);
  const float2* g = nat + gi * src_per;
  const long long row = 2LL * n1;
  const int my = (2 * n1 - ky) & (2 * n1 - 1);
  for (int i = threadIdx.x; i < 2 * n0 * kS3; i += blockDim.x) {
    const int kz = i / kS3, kb = i % kS3;
    if (kb >= nk) continue;
    const int kx = kb0 + kb;
    *HND_S(&tw[kz * (kS3 + 1) + kb]) = *HND_G(&g[(kz * row + ky) * pitch + kx]);
    if (pair) {
      const int mx = (2 * n2 - kx) & (2 * n2 - 1);
      *HND_S(&tm[kz * (kS3 + 1) + kb]) = *HND_G(&g[(kz * row + my) * pitch + mx]);
    }
  }
  __syncthreads();
  const int G = lanes_of(n0);
  const int nch = pair ? static_cast<int>(min(2LL, C - 2 * gi)) : 1;
  for (int i = threadIdx.x; i < nch * n0 * kS3; i += blockDim.x) {
    const int ch = i / (n0 * kS3), kb = (i / n0) % kS3, m = i % n0;
    if (kb >= nk) continue;
    const int f = spec_idx_gen(n0, m % G, m / G);
    float2 s2[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int kz = 2 * f + h;
      const float2 w = *HND_S(&tw[kz * (kS3 + 1) + kb]);
      if (!pair) {
        s2[h] = w;
      } else {
        const float2 wm = *HND_S(&tm[((2 * n0 - kz) & (2 * n0 - 1)) * (kS3 + 1) + kb]);
        s2[h] = ch ? make_float2(0.5f * (w.y + wm.y), 0.5f * (wm.x - w.x))
                   : make_float2(0.5f * (w.x + wm.x), 0.5f * (w.y - wm.y));
      }
    }
    const long long c = pair ? 2 * gi + ch : gi;
    const long long e = ((c * (n2 + 1) + kb0 + kb) * (2LL * n1) + ky) * n0 + m;
    *HND_G(&out[e]) = make_float4(scale * s2[0].x, scale * s2[1].x, scale * s2[0].y, scale * s2[1].y);
  }
}

static __global__ void k_spec3_out(const float4* __restrict__ lib, float2* __restrict__ nat, int n0, int n1, int n2,
                                   long long C) {
  const long long per = static_cast<long long>(n2 + 1) * 2 * n1 * n0;
  const int G = lanes_of(n0);
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < per * C;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long c = e / per, r = e % per;
    const int kx = static_cast<int>(r / (2LL * n1 * n0));
    const long long r2 = r % (2LL * n1 * n0);
    const int ky = static_cast<int>(r2 / n0), m = static_cast<int>(r2 % n0);
    const int f = spec_idx_gen(n0, m % G, m / G);
    float2* dst = nat + c * per * 2;
    const float4 v = *HND_G(&lib[e]);
    *HND_G(&dst[((2LL * f) * (2 * n1) + ky) * (n2 + 1) + kx]) = make_float2(v.x, v.z);
    *HND_G(&dst[((2LL * f + 1) * (2 * n1) + ky) * (n2 + 1) + kx]) = make_float2(v.y, v.w);
  }
}

}  // namespace hnd2
