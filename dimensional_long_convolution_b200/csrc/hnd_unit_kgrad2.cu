// Instantiations and launcher: the kernel-value gradient on the 2D
// multi-pass tier through the row-pair and half-spectrum stages
// (hnd_kgrad2.cuh), one chunk of channels at a time.
#include "hnd_host_util.h"
#include "hnd_kgrad2.cuh"
#include "hnd_launch.h"

namespace hnd {

namespace {

template <int N0>
cudaError_t kgcol_go(const float2* zu, const float2* zz, float2* zk, int n1, int B, int ncc, cudaStream_t st) {
  auto kern = hnd2::k_kgcol<N0>;
  const size_t sm = hnd2::KGC<N0>::kBytes;
  cudaError_t e = ensure_smem(kern, sm);
  if (e != cudaSuccess) return e;
  constexpr int UPB = hnd2::KGC<N0>::UPB;
  dim3 grid(ncc, (n1 - 1 + UPB - 1) / UPB);
  e = launch_pdl(true, kern, grid, dim3(hnd2::kTM), sm, st, zu, zz, zk, n1, B);
  if (e != cudaSuccess) return e;
  auto kdc = hnd2::k_kgcol_dc<N0>;
  const size_t smd = hnd2::KGCD<N0>::kBytes;
  if ((e = ensure_smem(kdc, smd)) != cudaSuccess) return e;
  return launch_pdl(true, kdc, dim3(ncc), dim3(32), smd, st, zu, zz, zk, n1, B);
}

template <int NL>
cudaError_t kginv_go(const float2* zk, float* dK, int n0, int ncc, int c0, float scale, cudaStream_t st) {
  auto kern = hnd2::k_kginv<NL>;
  const size_t sm = hnd2::RT<NL>::kBytes;
  cudaError_t e = ensure_smem(kern, sm);
  if (e != cudaSuccess) return e;
  constexpr int RPB = hnd2::RT<NL>::RPB;
  dim3 grid(ncc, (n0 + RPB - 1) / RPB);
  return launch_pdl(true, kern, grid, dim3(hnd2::kTM), sm, st, zk, dK, n0, c0, scale);
}

#define HND_SW(FN, N, ...)                  \
  switch (N) {                              \
    case 8: return FN<8>(__VA_ARGS__);      \
    case 16: return FN<16>(__VA_ARGS__);    \
    case 32: return FN<32>(__VA_ARGS__);    \
    case 64: return FN<64>(__VA_ARGS__);    \
    case 128: return FN<128>(__VA_ARGS__);  \
    case 256: return FN<256>(__VA_ARGS__);  \
    default: return cudaErrorInvalidValue;  \
  }

cudaError_t kgcol_n0(int n0, const float2* zu, const float2* zz, float2* zk, int n1, int B, int ncc,
                     cudaStream_t st) {
  HND_SW(kgcol_go, n0, zu, zz, zk, n1, B, ncc, st)
}

cudaError_t kginv_n1(int n1, const float2* zk, float* dK, int n0, int ncc, int c0, float scale, cudaStream_t st) {
  HND_SW(kginv_go, n1, zk, dK, n0, ncc, c0, scale, st)
}

}  // namespace

// One chunk of channels [c0, c0 + ncc) of a 2D problem on the multi-pass tier:
// forward rows of u = k v and z = q dy, column units with the batch sum, full
// inverse rows with the offset read-out.  `grids` holds 2 B ncc volumes of
// packed row spectra (u then z) and ncc channel grids (8 n0 n1 and 16 n0 n1
// bytes each).  4 + 1 launches.
cudaError_t launch_kgrad2d_chunk(const KgradLaunch& g, cudaStream_t st) {
  const int n0 = g.n[0], n1 = g.n[1];
  const long long zvol = static_cast<long long>(n0) * n1;              // float2 per volume
  const int nv = g.ncc * g.B;
  float2* zu = g.grids;
  float2* zz = zu + zvol * nv;
  float2* zk = zz + zvol * nv;
  ConvArgs a{};
  a.B = g.B;
  a.C = g.C;
  a.bf16 = g.bf16;
  a.ndim = 2;
  a.n[0] = n0;
  a.n[1] = n1;
  a.n[2] = 1;
  a.stream = st;
  const long long ord0 = static_cast<long long>(g.c0) * g.B;
  a.k = g.k, a.v = g.v;
  cudaError_t e = launch_rowfwd(a, n1, zu, ord0, nv, n0 / 2);
  a.k = g.q, a.v = g.dy;
  if (e == cudaSuccess) e = launch_rowfwd(a, n1, zz, ord0, nv, n0 / 2);
  if (e == cudaSuccess) e = kgcol_n0(n0, zu, zz, zk, n1, g.B, g.ncc, st);
  const float scale = static_cast<float>(1.0 / (4.0 * n0 * n1));
  if (e == cudaSuccess) e = kginv_n1(n1, zk, g.dK, n0, g.ncc, g.c0, scale, st);
  return e;
}

}  // namespace hnd
