// Instantiations: 1D fused rows, multi-pass row stages.
#include "hnd_kernels.cuh"
#include "hnd_multi2.cuh"
#include "hnd_launch.h"
#include "hnd_host_util.h"

namespace hnd {

template <int N, class IO, bool DUAL>
static cudaError_t rows1d_launch(const ConvArgs& a) {
  using TT = typename IO::T;
  auto kern = k_rows1d<N, IO, DUAL>;
  const size_t sm = kMidSmemBase;
  cudaError_t e = ensure_smem(kern, sm);
  if (e != cudaSuccess) return e;
  constexpr int PPW = 32 / (N / 8);
  const long long rpairs = (static_cast<long long>(a.B) * a.C + 1) / 2;
  long long blocks = (rpairs + kWarps * PPW - 1) / (kWarps * PPW);
  if (blocks > 148LL * 64) blocks = 148LL * 64;
  kern<<<static_cast<unsigned>(blocks), kThreads, sm, a.stream>>>(
      static_cast<const TT*>(a.q), static_cast<const TT*>(a.k), static_cast<const TT*>(a.v),
      static_cast<const float2*>(a.spec), a.sbs, static_cast<TT*>(a.y), a.B, a.C, a.sconj,
      static_cast<const TT*>(a.g2), static_cast<TT*>(a.y2));
  return cudaGetLastError();
}

template <int N, class IO>
static cudaError_t rows1d_go(const ConvArgs& a) {
  return a.y2 ? rows1d_launch<N, IO, true>(a) : rows1d_launch<N, IO, false>(a);
}

template <class IO>
static cudaError_t rows1d_io(const ConvArgs& a) {
  switch (a.n[0]) {
    case 8: return rows1d_go<8, IO>(a);
    case 16: return rows1d_go<16, IO>(a);
    case 32: return rows1d_go<32, IO>(a);
    case 64: return rows1d_go<64, IO>(a);
    case 128: return rows1d_go<128, IO>(a);
    case 256: return rows1d_go<256, IO>(a);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_rows1d(const ConvArgs& a) { return a.bf16 ? rows1d_io<IOBF16>(a) : rows1d_io<IOF32>(a); }

template <class IO>
struct TypeOf;
template <>
struct TypeOf<IOF32> {
  using T = float;
};
template <>
struct TypeOf<IOBF16> {
  using T = __nv_bfloat16;
};

static int pair_stride(const ConvArgs& a) { return a.ndim == 2 ? a.n[0] / 2 : 1; }

template <int NL, class IO>
static cudaError_t rowfwd_go(const ConvArgs& a, float2* zt, long long ord0, int np, int rp_total) {
  using TT = typename TypeOf<IO>::T;
  auto kern = hnd2::k_rowfwd2<NL, TT>;
  const size_t sm = hnd2::RT<NL>::kBytes;
  cudaError_t e = ensure_smem(kern, sm);
  if (e != cudaSuccess) return e;
  constexpr int RPB = hnd2::RT<NL>::RPB;
  dim3 grid(np, (rp_total + RPB - 1) / RPB);
  return launch_pdl(true, kern, grid, dim3(hnd2::kTM), sm, a.stream, static_cast<const TT*>(a.k),
                    static_cast<const TT*>(a.v), zt, ord0, rp_total, pair_stride(a), a.B, a.C);
}

template <int NL, class IO>
static cudaError_t rowinv_go(const ConvArgs& a, const float2* zt, long long ord0, int np, int rp_total) {
  using TT = typename TypeOf<IO>::T;
  auto kern = hnd2::k_rowinv2<NL, TT>;
  const size_t sm = hnd2::RT<NL>::kBytes;
  cudaError_t e = ensure_smem(kern, sm);
  if (e != cudaSuccess) return e;
  constexpr int RPB = hnd2::RT<NL>::RPB;
  dim3 grid(np, (rp_total + RPB - 1) / RPB);
  // Early launch after the 3D slab kernel measured slower (its CTAs crowd the
  // slab kernel's tail); after the 2D column kernel it pays.
  return launch_pdl(a.ndim == 2, kern, grid, dim3(hnd2::kTM), sm, a.stream, zt, static_cast<const TT*>(a.q),
                    static_cast<TT*>(a.y), ord0, rp_total, pair_stride(a), a.B, a.C,
                    static_cast<const TT*>(a.g2), static_cast<TT*>(a.y2));
}

#define HND_ROWS_SWITCH(FN, IO, ...)                  \
  switch (nl) {                                       \
    case 8: return FN<8, IO>(__VA_ARGS__);            \
    case 16: return FN<16, IO>(__VA_ARGS__);          \
    case 32: return FN<32, IO>(__VA_ARGS__);          \
    case 64: return FN<64, IO>(__VA_ARGS__);          \
    case 128: return FN<128, IO>(__VA_ARGS__);        \
    case 256: return FN<256, IO>(__VA_ARGS__);        \
    default: return cudaErrorInvalidValue;            \
  }

cudaError_t launch_rowfwd(const ConvArgs& a, int nl, float2* zt, long long ord0, int np, int rp_total) {
  if (a.bf16) {
    HND_ROWS_SWITCH(rowfwd_go, IOBF16, a, zt, ord0, np, rp_total)
  } else {
    HND_ROWS_SWITCH(rowfwd_go, IOF32, a, zt, ord0, np, rp_total)
  }
}

cudaError_t launch_rowinv(const ConvArgs& a, int nl, const float2* zt, long long ord0, int np, int rp_total) {
  if (a.bf16) {
    HND_ROWS_SWITCH(rowinv_go, IOBF16, a, zt, ord0, np, rp_total)
  } else {
    HND_ROWS_SWITCH(rowinv_go, IOF32, a, zt, ord0, np, rp_total)
  }
}

}  // namespace hnd
