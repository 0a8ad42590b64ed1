// Long 1D tier: one convolution over all channel pairs in waves, each wave the
// 2m - 1 fused passes of hnd_long1d.cuh over the split P = 2n = P0 P1 (P2).
#include "hnd_launch.h"
#include "hnd_host_util.h"
#include "hnd_long1d.cuh"

namespace hnd {

namespace {

template <int N, int KIND, class T, bool DUAL>
cudaError_t l1_pass_go(const hnd2::L1PassArgs& a, cudaStream_t st) {
  auto kern = hnd2::k_l1_pass<N, KIND, T, DUAL>;
  const size_t sm = hnd2::AxisSmem<N>::kBytes;
  cudaError_t e = ensure_smem(kern, sm);
  if (e != cudaSuccess) return e;
  const long long per_cta = (hnd2::kAT / 32) * (32 / hnd2::P2<N>::G);
  long long blocks = (a.npen + per_cta - 1) / per_cta;
  if (blocks > 148LL * 16) blocks = 148LL * 16;
  if (blocks < 1) blocks = 1;
  return launch_pdl(true, kern, dim3(static_cast<unsigned>(blocks)), dim3(hnd2::kAT), sm, st, a);
}

template <int N>
cudaError_t l1_center_go(const hnd2::L1PassArgs& a, cudaStream_t st) {
  auto kern = hnd2::k_l1_center<N>;
  const size_t sm = hnd2::AxisSmem<N>::kBytes;
  cudaError_t e = ensure_smem(kern, sm);
  if (e != cudaSuccess) return e;
  const long long per_cta = (hnd2::kAT / 32) * (32 / hnd2::P2<N>::G / 2);
  long long blocks = (a.npen + per_cta - 1) / per_cta;
  if (blocks > 148LL * 16) blocks = 148LL * 16;
  if (blocks < 1) blocks = 1;
  return launch_pdl(true, kern, dim3(static_cast<unsigned>(blocks)), dim3(hnd2::kAT), sm, st, a);
}

cudaError_t l1_center(int N, const hnd2::L1PassArgs& a, cudaStream_t st) {
  switch (N) {
    case 16: return l1_center_go<16>(a, st);
    case 32: return l1_center_go<32>(a, st);
    case 64: return l1_center_go<64>(a, st);
    case 128: return l1_center_go<128>(a, st);
    case 256: return l1_center_go<256>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

template <int N, bool INV>
cudaError_t l1_mid_go(const hnd2::L1PassArgs& a, cudaStream_t st) {
  auto kern = hnd2::k_l1_mid2g<N, INV>;
  const size_t sm = hnd2::AxisSmem<N>::kBytes;
  cudaError_t e = ensure_smem(kern, sm);
  if (e != cudaSuccess) return e;
  const long long per_cta = 2 * (hnd2::kAT / 32) * (32 / hnd2::P2<N>::G);   // two pencil groups
  long long blocks = (a.npen + per_cta - 1) / per_cta;
  if (blocks > 148LL * 16) blocks = 148LL * 16;
  if (blocks < 1) blocks = 1;
  return launch_pdl(true, kern, dim3(static_cast<unsigned>(blocks)), dim3(hnd2::kAT), sm, st, a);
}

template <int KIND, class T, bool DUAL>
cudaError_t l1_pass(int N, const hnd2::L1PassArgs& a, cudaStream_t st);

// a middle pass: the two-group kernel for 8-slot pencils, else k_l1_pass
template <bool INV>
cudaError_t l1_mid(int N, const hnd2::L1PassArgs& a, cudaStream_t st) {
  switch (N) {
    case 16: return l1_mid_go<16, INV>(a, st);
    case 32: return l1_mid_go<32, INV>(a, st);
    case 64: return l1_mid_go<64, INV>(a, st);
    default:
      return INV ? l1_pass<hnd2::kInvMid, float, false>(N, a, st) : l1_pass<hnd2::kFwdMid, float, false>(N, a, st);
  }
}

template <int KIND, class T, bool DUAL>
cudaError_t l1_pass(int N, const hnd2::L1PassArgs& a, cudaStream_t st) {
  switch (N) {
    case 16: return l1_pass_go<16, KIND, T, DUAL>(a, st);
    case 32: return l1_pass_go<32, KIND, T, DUAL>(a, st);
    case 64: return l1_pass_go<64, KIND, T, DUAL>(a, st);
    case 128: return l1_pass_go<128, KIND, T, DUAL>(a, st);
    case 256: return l1_pass_go<256, KIND, T, DUAL>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

int ilog2(long long x) {
  int l = 0;
  while ((1LL << l) < x) ++l;
  return l;
}

// One wave: `cnt` channel-pair grids from pair v0.  part 0: the first pass
// only; part 1: the rest; part 2: all of it.
template <class T>
cudaError_t long1d_t(const ConvArgs& c, float2* grid, long long v0, long long cnt, int part, int* launches) {
  const L1Split sp = long1d_split(c.n[0]);
  const int m = sp.m;
  const long long P = 2LL * c.n[0];
  long long stride[3] = {1, 1, 1};
  for (int a = m - 2; a >= 0; --a) stride[a] = stride[a + 1] * sp.P[a + 1];
  hnd2::L1PassArgs a{};
  a.grid = grid;
  a.P = P;
  a.lgP = ilog2(P);
  a.n = c.n[0];
  a.H = (c.C + 1) / 2;
  a.a = c.k;
  a.b = c.v;
  a.q = c.q;
  a.y = c.y;
  a.g2 = c.g2;
  a.y2 = c.y2;
  a.spec = static_cast<const float4*>(c.spec);
  a.sbs4 = c.sbs / 2;
  a.sd = hnd2::l1_spec_of(m, sp.P);
  a.lgP0 = ilog2(sp.P[0]);
  a.sconj = c.sconj;
  a.C = c.C;
  a.v0 = v0;
  auto set_axis = [&](int ax) {
    a.stride = stride[ax];
    a.lgS = ilog2(stride[ax]);
    a.npen = cnt * P / sp.P[ax];
  };
  cudaError_t e = cudaSuccess;
  if (part != 1) {
    // forward: axis 0 from k v
    set_axis(0);
    a.twQ = P;
    a.lgQ = ilog2(a.twQ);
    e = l1_pass<hnd2::kFirst, T, false>(sp.P[0] / 2, a, c.stream);
    *launches += 1;
    if (part == 0 || e != cudaSuccess) return e;
  }
  if (m == 3) {
    // forward axis 1 (three levels)
    set_axis(1);
    a.twQ = static_cast<long long>(sp.P[1]) * sp.P[2];
    a.lgQ = ilog2(a.twQ);
    e = l1_mid<false>(sp.P[1] / 2, a, c.stream);
  }
  // spectrum product on the last axis, pencil pairs, with the inverse
  // transform back
  if (e == cudaSuccess) {
    set_axis(m - 1);
    a.npen = cnt * a.sd.R;
    a.twP = sp.P[m - 2];
    a.twQ = static_cast<long long>(sp.P[m - 2]) * sp.P[m - 1];
    a.lgQ = ilog2(a.twQ);
    e = l1_center(sp.P[m - 1] / 2, a, c.stream);
  }
  if (e == cudaSuccess && m == 3) {
    set_axis(1);
    a.twP = sp.P[0];
    a.twQ = P;
    a.lgQ = ilog2(a.twQ);
    e = l1_mid<true>(sp.P[1] / 2, a, c.stream);
  }
  if (e == cudaSuccess) {
    set_axis(0);
    e = c.y2 ? l1_pass<hnd2::kLast, T, true>(sp.P[0] / 2, a, c.stream)
             : l1_pass<hnd2::kLast, T, false>(sp.P[0] / 2, a, c.stream);
  }
  *launches += 2 * m - 2;
  return e;
}

}  // namespace

int long1d_conv_launches(int n) { return 2 * long1d_split(n).m - 1; }

cudaError_t launch_long1d_wave(const ConvArgs& a, float2* grid, long long v0, long long cnt, int part,
                               int* launches) {
  return a.bf16 ? long1d_t<__nv_bfloat16>(a, grid, v0, cnt, part, launches)
                : long1d_t<float>(a, grid, v0, cnt, part, launches);
}

cudaError_t launch_long1d(const ConvArgs& a, float2* grid, long long wave, int* launches) {
  const long long grids = static_cast<long long>(a.B) * ((a.C + 1) / 2);
  cudaError_t e = cudaSuccess;
  for (long long v0 = 0; v0 < grids && e == cudaSuccess; v0 += wave)
    e = launch_long1d_wave(a, grid, v0, grids - v0 < wave ? grids - v0 : wave, 2, launches);
  return e;
}

}  // namespace hnd
