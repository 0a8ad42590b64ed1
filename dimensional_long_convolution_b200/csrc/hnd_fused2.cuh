// hnd_fused2.cuh -- persistent fused 2D tier on the packed two-path FFT core.
//
// One CTA (256 threads, two per SM) walks (b, c) volumes.  Per volume, all
// in shared memory (HyenaND arXiv summary, "Implementation: nSubQ": forward
// FFT, spectral modulation, inverse FFT and output cropping fused, with the
// intermediates on chip):
//   stage 1  rows r and r + n0/2 packed as one complex row, zero-padded
//            forward transform along axis 1 -> Zb[kk][rp]
//   stage 2  per last-axis frequency: unpack both rows, zero-padded
//            convolution along axis 0 with the channel spectrum, repack
//   stage 3  inverse row transforms, crop, output gate q, store y
// k and v of the next volume are prefetched with bulk asynchronous copies
// (one per row, into a padded staging pitch) while stages 2-3 run.
#pragma once

#include "hnd_fft2.cuh"

namespace hnd2 {

static __device__ const float2 g_tw512[512] =
#include "hnd_twiddles.inc"
;

constexpr int kT = 256;          // threads per CTA
constexpr int kW = kT / 32;      // warps per CTA

// ------------------------------------------------------- async copy (TMA)
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

// Bounded wait on a phase of an mbarrier: gives up after about `limit`
// cycles, records a timeout in the status word and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, unsigned parity, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  const long long limit = 4000000000LL;     // about 2 s at 2 GHz
  for (long long it = 0; it < (1LL << 28); ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if (clock64() - t0 > limit) break;
  }
  if (status) atomicCAS(status, 0, 6 /* HYENA_ND_ERR_DEVICE_TIMEOUT */);
  return false;
}

// ------------------------------------------------------------ activations
template <class T>
struct Act;
template <>
struct Act<float> {
  static __device__ __forceinline__ float ld_s(const float* p) { return *HND_S(p); }
  static __device__ __forceinline__ float ld_g(const float* p) { return __ldcs(HND_G(p)); }
  static __device__ __forceinline__ void st_g(float* p, float x) { __stcs(HND_G(p), x); }
};
template <>
struct Act<__nv_bfloat16> {
  static __device__ __forceinline__ float ld_s(const __nv_bfloat16* p) {
    return __uint_as_float(static_cast<unsigned>(*HND_S(reinterpret_cast<const unsigned short*>(p))) << 16);
  }
  static __device__ __forceinline__ float ld_g(const __nv_bfloat16* p) {
    return __uint_as_float(static_cast<unsigned>(__ldcs(HND_G(reinterpret_cast<const unsigned short*>(p)))) << 16);
  }
  static __device__ __forceinline__ void st_g(__nv_bfloat16* p, float x) {
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    __stcs(HND_G(reinterpret_cast<unsigned short*>(p)), *reinterpret_cast<const unsigned short*>(&h));
  }
};

// ------------------------------------------------------------ the kernel
// 512 threads = two groups of 8 warps.  Volumes are software-pipelined with
// two Zb buffers: in phase A group 0 finishes volume i (inverse rows, crop,
// gate, store) while group 1 starts volume i+1 (forward rows); in phase B all
// 16 warps run the column stage of volume i+1.  Two barriers per volume and
// every warp busy in both phases.  k, v (for the forward rows) and q (for the
// output gate) arrive by bulk asynchronous copies one phase ahead.
constexpr int kT3 = 512;
constexpr int kW3 = kT3 / 32;

template <int N0, int N1, class T>
struct F3 {
  static constexpr int PITCH = (N1 * static_cast<int>(sizeof(T)) / 4 + 8) * 4 / static_cast<int>(sizeof(T));
  static constexpr int RPS = N0 / 2 + 1;                 // Zb pitch (float2) per frequency row
  static constexpr size_t kTabs = Tabs<N0>::kBytes + (N0 == N1 ? 0 : Tabs<N1>::kBytes);
  static constexpr size_t kStage = static_cast<size_t>(N0) * PITCH * sizeof(T);   // one plane
  static constexpr size_t kZb = sizeof(float4) * N1 * RPS;    // [f][rp] float4
  static constexpr int XW = XB<N0>::kWarp > XB<N1>::kWarp ? XB<N0>::kWarp : XB<N1>::kWarp;
  static constexpr size_t kX = 16ull * XW * kW3;
  static constexpr size_t kBytes = 32 + kTabs + 3 * kStage + 2 * kZb + kX;
};

// Row-stage work of one warp group (8 warps): forward rows of a volume.
template <int N0, int N1, class T>
__device__ __forceinline__ void rows_fwd(const T* kst, const T* vst, float4* Zb, float4* xb, Tabs<N1> t1, int gw,
                                         int lane) {
  using L = F3<N0, N1, T>;
  constexpr int G = P2<N1>::G, PPW = 32 / G;
  const int pen = lane / G, g = lane % G;
  const unsigned mask = pmask<N1>(lane);
  const int key = pkey<N1>(pen);
  float4* buf = xb + pen * XB<N1>::kPen;
  for (int r0 = gw * PPW; r0 < N0 / 2; r0 += 8 * PPW) {
    const int rp = r0 + pen;
    const bool act = rp < N0 / 2;
    float2 z[8];
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const int j = g + s * G;
      const int ra = rp * L::PITCH + j, rb = (rp + N0 / 2) * L::PITCH + j;
      z[s] = act ? make_float2(Act<T>::ld_s(kst + ra) * Act<T>::ld_s(vst + ra),
                               Act<T>::ld_s(kst + rb) * Act<T>::ld_s(vst + rb))
                 : make_float2(0.f, 0.f);
    }
    cp x[8];
    padded_fwd<N1>(z, x, g, buf, key, t1, mask);
    if (act) {
#pragma unroll
      for (int s = 0; s < 8; ++s)
        *HND_S(&Zb[spec_idx<N1>(g, s) * L::RPS + rp]) = make_float4(x[s].re.x, x[s].im.x, x[s].re.y, x[s].im.y);
    }
  }
}

// Inverse rows, crop, output gate and store of one volume (8 warps).
template <int N0, int N1, class T, bool DUAL>
__device__ __forceinline__ void rows_inv(const T* qst, const float4* Zb, T* yp, float4* xb, Tabs<N1> t1, int gw,
                                         int lane, const T* __restrict__ g2p, T* __restrict__ y2p) {
  using L = F3<N0, N1, T>;
  constexpr int G = P2<N1>::G, PPW = 32 / G;
  const int pen = lane / G, g = lane % G;
  const unsigned mask = pmask<N1>(lane);
  const int key = pkey<N1>(pen);
  float4* buf = xb + pen * XB<N1>::kPen;
  for (int r0 = gw * PPW; r0 < N0 / 2; r0 += 8 * PPW) {
    const int rp = r0 + pen;
    const bool act = rp < N0 / 2;
    cp x[8];
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const float4 e = act ? *HND_S(&Zb[spec_idx<N1>(g, s) * L::RPS + rp]) : make_float4(0.f, 0.f, 0.f, 0.f);
      x[s] = {make_float2(e.x, e.z), make_float2(e.y, e.w)};
    }
    float2 o[8];
    padded_inv<N1>(x, o, g, buf, key, t1, mask);
    if (act) {
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const int j = g + s * G;
        const float qa = Act<T>::ld_s(qst + rp * L::PITCH + j);
        const float qb = Act<T>::ld_s(qst + (rp + N0 / 2) * L::PITCH + j);
        Act<T>::st_g(yp + static_cast<long long>(rp) * N1 + j, o[s].x * qa);
        Act<T>::st_g(yp + static_cast<long long>(rp + N0 / 2) * N1 + j, o[s].y * qb);
      }
      if constexpr (DUAL) {      // second gated output of the same convolution
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          const long long ja = static_cast<long long>(rp) * N1 + g + s * G;
          const long long jb = ja + static_cast<long long>(N0 / 2) * N1;
          Act<T>::st_g(y2p + ja, o[s].x * Act<T>::ld_g(g2p + ja));
          Act<T>::st_g(y2p + jb, o[s].y * Act<T>::ld_g(g2p + jb));
        }
      }
    }
  }
}

// Column stage of one volume by all 16 warps.  Unit cu = last-axis frequency
// kx (cu >= 1) or the combined DC/Nyquist unit (cu = 0).  Zb holds, per
// half-frequency f and row pair, the two padded frequencies 2f and 2f+1 side
// by side, so frequency kx lives at float2 (f RPS + rp) 2 + (kx & 1); the
// pencils of a warp take adjacent units, which puts the two pencils of a
// 16-lane phase on opposite bank parities.  The warp that owns unit 0 runs the
// general product A Z + B conj(Z[-k]) for all its pencils so it does not
// diverge.
template <int N0, int N1, class T>
__device__ __forceinline__ void columns(float4* Zb4, float4* xb, const float4* __restrict__ sp, Tabs<N0> t0,
                                        int warp, int lane, float sgn) {
  using L = F3<N0, N1, T>;
  constexpr int G = P2<N0>::G, PPW = 32 / G;
  constexpr int SLOTS = kW3 * PPW;
  float2* Zb = reinterpret_cast<float2*>(Zb4);
  const int pen = lane / G, g = lane % G;
  const unsigned mask = pmask<N0>(lane);
  const int key = pkey<N0>(pen);
  float4* buf = xb + pen * XB<N0>::kPen;
  const int sidx = warp * PPW + pen;
  auto zidx = [](int kk, int rp) { return ((kk >> 1) * L::RPS + rp) * 2 + (kk & 1); };
  for (int round = 0; round * SLOTS < N1; ++round) {
    const int cu = round * SLOTS + sidx;
    const bool act = cu < N1;
    const bool general = round == 0 && warp == 0;      // this warp holds unit 0
    const int kx = cu, kxm = cu == 0 ? N1 : 2 * N1 - cu;
    float4 S[8];
    if (act) {
      const float4* su = sp + (cu == 0 ? 0LL : static_cast<long long>(cu + 1) * N0);
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        S[s] = __ldg(HND_G(su + s * G + g));
        S[s].z *= sgn, S[s].w *= sgn;     // sgn = -1: conjugate spectrum (adjoint)
      }
    }
    float2 z[8];
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int rp = g + s * G;
      float2 z1 = make_float2(0.f, 0.f), z2 = z1;
      if (act) {
        z1 = *HND_S(&Zb[zidx(kx, rp)]);
        z2 = *HND_S(&Zb[zidx(kxm, rp)]);
      }
      if (cu == 0) {
        z[s] = make_float2(z1.x, z2.x);       // row a: (DC, Nyquist)
        z[s + 4] = make_float2(z1.y, z2.y);   // row b
      } else {
        z[s] = unpack_a(z1, z2);
        z[s + 4] = unpack_b(z1, z2);
      }
    }
    cp x[8];
    padded_fwd<N0>(z, x, g, buf, key, t0, mask);
    if (general) {
      cp xp[8];
      fetch_partner<N0>(x, xp, g, buf, key, mask);
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        float4 Bc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (cu == 0) {
          Bc = __ldg(HND_G(sp + N0 + s * G + g));
          Bc.z *= sgn, Bc.w *= sgn;
        }
        const cp a = cmulp(x[s], make_float2(S[s].x, S[s].y), make_float2(S[s].z, S[s].w));
        const cp xc = {xp[s].re, make_float2(-xp[s].im.x, -xp[s].im.y)};
        const cp bb = cmulp(xc, make_float2(Bc.x, Bc.y), make_float2(Bc.z, Bc.w));
        x[s] = cadd(a, bb);
      }
    } else if (act) {
#pragma unroll
      for (int s = 0; s < 8; ++s) x[s] = cmulp(x[s], make_float2(S[s].x, S[s].y), make_float2(S[s].z, S[s].w));
    }
    float2 o[8];
    padded_inv<N0>(x, o, g, buf, key, t0, mask);
    if (act) {
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const int rp = g + s * G;
        const float2 ya = o[s], yb = o[s + 4];
        if (cu == 0) {
          *HND_S(&Zb[zidx(0, rp)]) = make_float2(ya.x, yb.x);
          *HND_S(&Zb[zidx(N1, rp)]) = make_float2(ya.y, yb.y);
        } else {
          *HND_S(&Zb[zidx(kx, rp)]) = pack_pos(ya, yb);
          *HND_S(&Zb[zidx(kxm, rp)]) = pack_neg(ya, yb);
        }
      }
    }
  }
}

__device__ __forceinline__ void named_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ void named_arrive(int id, int nthreads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

template <int N0, int N1, class T, bool DUAL>
__global__ void __launch_bounds__(kT3, 1)
    k_fused2d_v3(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                 const float4* __restrict__ spec, long long sbs4, T* __restrict__ y, int B, int C, int* status,
                 float sgn, const T* __restrict__ g2, T* __restrict__ y2) {
  using L = F3<N0, N1, T>;
  extern __shared__ __align__(16) unsigned char smem[];
  uint64_t* bar_kv = reinterpret_cast<uint64_t*>(smem);
  uint64_t* bar_q = bar_kv + 1;
  unsigned char* p = smem + 32;
  const Tabs<N0> t0 = tabs_at<N0>(p);
  Tabs<N1> t1;
  if constexpr (N0 == N1) {
    t1 = t0;
  } else {
    t1 = tabs_at<N1>(p + Tabs<N0>::kBytes);
  }
  p += L::kTabs;
  T* kst = reinterpret_cast<T*>(p);
  T* vst = reinterpret_cast<T*>(p + L::kStage);
  T* qst = reinterpret_cast<T*>(p + 2 * L::kStage);
  float4* Zb0 = reinterpret_cast<float4*>(p + 3 * L::kStage);
  float4* Zb1 = reinterpret_cast<float4*>(p + 3 * L::kStage + L::kZb);
  float4* xb = reinterpret_cast<float4*>(p + 3 * L::kStage + 2 * L::kZb);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = warp >> 3, gw = warp & 7;
  float4* xw = xb + warp * L::XW;
  const int nvol = B * C;
  const int v0 = blockIdx.x;
  if (v0 >= nvol) return;
  constexpr long long Lv = static_cast<long long>(N0) * N1;

  tabs_build<N0>(t0, g_tw512);
  if constexpr (N0 != N1) tabs_build<N1>(t1, g_tw512);

  auto vol_base = [&](int vv) {
    const int cc = vv / B, bb = vv % B;
    return (static_cast<long long>(bb) * C + cc) * Lv;
  };
  // Bulk row copies, one row per thread.  Every copying thread first arrives
  // on the barrier with the bytes it will deliver (barrier counts: 2 N0 for
  // k and v, N0 for q), so a phase completes only when all rows have landed.
  // Copies are only issued after a CTA barrier that follows the previous
  // phase's completion and the last reads of the staging buffer.
  auto copy_kv = [&](int vv) {
    const long long base = vol_base(vv);
    const int r = threadIdx.x;
    if (r < 2 * N0) {
      const int row = r % N0;
      const T* src = (r < N0 ? k : v) + base + static_cast<long long>(row) * N1;
      T* dst = (r < N0 ? kst : vst) + row * L::PITCH;
      // (checked build: a copy outside its buffers is skipped and delivers no bytes)
      const bool okc = HND_RANGE_OK(src, N1 * sizeof(T)) && HND_RANGE_OK(dst, N1 * sizeof(T));
      fence_proxy_async();
      mbar_expect_tx(bar_kv, okc ? N1 * sizeof(T) : 0u);
      if (okc) bulk_g2s(dst, src, N1 * sizeof(T), bar_kv);
    }
  };
  auto copy_q = [&](int vv) {
    const long long base = vol_base(vv);
    const int r = threadIdx.x;
    if (r < N0) {
      const T* src = q + base + static_cast<long long>(r) * N1;
      T* dst = qst + r * L::PITCH;
      const bool okc = HND_RANGE_OK(src, N1 * sizeof(T)) && HND_RANGE_OK(dst, N1 * sizeof(T));
      fence_proxy_async();
      mbar_expect_tx(bar_q, okc ? N1 * sizeof(T) : 0u);
      if (okc) bulk_g2s(dst, src, N1 * sizeof(T), bar_q);
    }
  };

  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 2 * N0);
    mbar_init(bar_q, N0);
    fence_mbar_init();
  }
  __syncthreads();
  copy_kv(v0);
  copy_q(v0);
  unsigned ph_kv = 0, ph_q = 0;
  bool ok = true;

  // prologue: forward rows of the first volume by group 1
  if (grp == 1) {
    ok = mbar_wait_bounded(bar_kv, ph_kv, status);
    if (ok) rows_fwd<N0, N1, T>(kst, vst, Zb0, xw, t1, gw, lane);
  }
  int vol = v0;
  int next = vol + gridDim.x;
  if (!__syncthreads_and(ok)) {
    // a copy never arrived: one more bounded wait for the copies in flight, then stop
    mbar_wait_bounded(bar_kv, ph_kv, nullptr);
    mbar_wait_bounded(bar_q, ph_q, nullptr);
    return;
  }
  ph_kv ^= 1u;
  if (next < nvol) copy_kv(next);

  for (int i = 0; vol < nvol; ++i, vol = next, next += gridDim.x) {
    const int c = vol / B, b = vol % B;
    float4* Zc = (i & 1) ? Zb1 : Zb0;
    float4* Zn = (i & 1) ? Zb0 : Zb1;
    const float4* sp = spec + static_cast<long long>(b) * sbs4 + static_cast<long long>(c) * (N1 + 1) * N0;

    // phase B: columns of `vol`.  Group 0 needs every column before its
    // inverse rows; group 1 only signals and goes on to the next volume's
    // forward rows (they touch the other Zb buffer and the staging planes).
    columns<N0, N1, T>(Zc, xw, sp, t0, warp, lane, sgn);
    if (grp == 0) named_sync(1, kT3);
    else named_arrive(1, kT3);

    // phase A: group 0 finishes `vol`, group 1 starts `next`
    ok = true;
    if (grp == 0) {
      ok = mbar_wait_bounded(bar_q, ph_q, status);
      if (ok) {
        const long long vo = (static_cast<long long>(b) * C + c) * Lv;
        rows_inv<N0, N1, T, DUAL>(qst, Zc, y + vo, xw, t1, gw, lane, g2 + vo, y2 + vo);
      }
    } else if (next < nvol) {
      ok = mbar_wait_bounded(bar_kv, ph_kv, status);
      if (ok) rows_fwd<N0, N1, T>(kst, vst, Zn, xw, t1, gw, lane);
    }
    const int next2 = next + gridDim.x;
    if (!__syncthreads_and(ok)) {
      // a copy never arrived: one more bounded wait for the copies in flight, then stop
      mbar_wait_bounded(bar_q, ph_q, nullptr);
      if (next < nvol) mbar_wait_bounded(bar_kv, ph_kv, nullptr);
      return;
    }
    ph_q ^= 1u;
    if (next < nvol) ph_kv ^= 1u;
    if (next < nvol) copy_q(next);
    if (next2 < nvol) copy_kv(next2);
  }
}

// ------------------------------------------------------ spectrum layout (2D)
// Library order of a 2D problem, per channel, in float4 units:
// unit 0 (DC and Nyquist columns combined) holds A then B, n0 float4 each;
// unit u >= 1 (column kx = u) holds n0 float4 at offset (u + 1) n0.  Inside a
// unit, float4 m = s G + g holds (S[2f].re, S[2f+1].re, S[2f].im, S[2f+1].im)
// with f = spec_idx(g, s) the z-pencil frequency of lane g, slot s.
__host__ __device__ __forceinline__ int spec_idx_rt(int N, int g, int s) {
  if (N == 8) return s;
  const int R1 = N >= 128 ? 16 : 8, G = N / R1;
  return g + G * (s / G) + (s % G) * R1;
}

struct Pos2 {
  int kind;      // 0 plain column, 1 = A (combined), 2 = B (combined)
  int kx;        // plain column index
  int ky0, ky1;  // padded frequencies held by path 0 and path 1
};

__host__ __device__ __forceinline__ Pos2 pos2_of(int n0, int n1, long long e4) {
  Pos2 r;
  long long m;
  if (e4 < 2LL * n0) {
    r.kind = 1 + static_cast<int>(e4 / n0);
    r.kx = 0;
    m = e4 % n0;
  } else {
    r.kind = 0;
    r.kx = static_cast<int>((e4 - 2LL * n0) / n0) + 1;
    m = (e4 - 2LL * n0) % n0;
  }
  const int G = n0 == 8 ? 1 : n0 / (n0 >= 128 ? 16 : 8);
  const int s = static_cast<int>(m / G), g = static_cast<int>(m % G);
  const int f = spec_idx_rt(n0, g, s);
  r.ky0 = 2 * f;
  r.ky1 = 2 * f + 1;
  return r;
}

// Value at (row ky, column kx) of channel c of a source: a natural array
// [C][2 n0][pitch], or (pair) the full grids of the filter call that hold two
// channels per complex grid, K_c + i K_{c+1} for even c, whose transform W
// gives S_c = (W[k] + conj W[-k]) / 2 and S_{c+1} = (W[k] - conj W[-k]) / (2i).
__device__ __forceinline__ float2 src2_at(const float2* __restrict__ nat, long long c, long long src_per,
                                          long long pitch, int ky, int kx, int n0, int n1, int pair) {
  if (!pair) return *HND_G(&nat[c * src_per + ky * pitch + kx]);
  const float2* g = nat + (c >> 1) * src_per;
  const float2 w = *HND_G(&g[ky * pitch + kx]);
  const float2 m = *HND_G(&g[static_cast<long long>((2 * n0 - ky) & (2 * n0 - 1)) * pitch + ((2 * n1 - kx) & (2 * n1 - 1))]);
  return (c & 1) ? make_float2(0.5f * (w.y + m.y), 0.5f * (m.x - w.x)) : make_float2(0.5f * (w.x + m.x), 0.5f * (w.y - m.y));
}

// natural half spectrum [C][2 n0][n1 + 1] (or the filter call's full grids,
// pitch 2 n1, pair: two channels per grid) -> library order (v2)
static __global__ void k_spec_import_v2(const float2* __restrict__ nat, float4* __restrict__ out, int n0, int n1,
                                 long long C, long long full_pitch, float scale, int pair = 0) {
  // full_pitch: row length of the source (n1 + 1 for a half spectrum, 2 n1 for a full grid)
  const long long per = static_cast<long long>(n1 + 1) * n0;         // float4 per channel
  const long long src_per = static_cast<long long>(2 * n0) * full_pitch;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < per * C;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long c = e / per, e4 = e % per;
    const Pos2 ps = pos2_of(n0, n1, e4);
    float2 s0, s1;
    if (ps.kind == 0) {
      s0 = src2_at(nat, c, src_per, full_pitch, ps.ky0, ps.kx, n0, n1, pair);
      s1 = src2_at(nat, c, src_per, full_pitch, ps.ky1, ps.kx, n0, n1, pair);
    } else {
      const float sg = ps.kind == 1 ? 1.f : -1.f;
      const float2 a0 = src2_at(nat, c, src_per, full_pitch, ps.ky0, 0, n0, n1, pair);
      const float2 b0 = src2_at(nat, c, src_per, full_pitch, ps.ky0, n1, n0, n1, pair);
      const float2 a1 = src2_at(nat, c, src_per, full_pitch, ps.ky1, 0, n0, n1, pair);
      const float2 b1 = src2_at(nat, c, src_per, full_pitch, ps.ky1, n1, n0, n1, pair);
      s0 = make_float2(0.5f * (a0.x + sg * b0.x), 0.5f * (a0.y + sg * b0.y));
      s1 = make_float2(0.5f * (a1.x + sg * b1.x), 0.5f * (a1.y + sg * b1.y));
    }
    *HND_G(&out[e]) = make_float4(scale * s0.x, scale * s1.x, scale * s0.y, scale * s1.y);
  }
}

// library order (v2) -> natural half spectrum [C][2 n0][n1 + 1]
static __global__ void k_spec_export_v2(const float4* __restrict__ lib, float2* __restrict__ nat, int n0, int n1,
                                 long long C) {
  const long long per = static_cast<long long>(n1 + 1) * n0;
  const long long W = n1 + 1;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < per * C;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long c = e / per, e4 = e % per;
    const Pos2 ps = pos2_of(n0, n1, e4);
    float2* dst = nat + c * per * 2;
    const float4 f = *HND_G(&lib[e]);
    if (ps.kind == 0) {
      *HND_G(&dst[ps.ky0 * W + ps.kx]) = make_float2(f.x, f.z);
      *HND_G(&dst[ps.ky1 * W + ps.kx]) = make_float2(f.y, f.w);
    } else if (ps.kind == 1) {
      const float4 g = *HND_G(&lib[e + n0]);     // the B payload at the same position
      *HND_G(&dst[ps.ky0 * W]) = make_float2(f.x + g.x, f.z + g.z);
      *HND_G(&dst[ps.ky0 * W + n1]) = make_float2(f.x - g.x, f.z - g.z);
      *HND_G(&dst[ps.ky1 * W]) = make_float2(f.y + g.y, f.w + g.w);
      *HND_G(&dst[ps.ky1 * W + n1]) = make_float2(f.y - g.y, f.w - g.w);
    }
  }
}

}  // namespace hnd2
