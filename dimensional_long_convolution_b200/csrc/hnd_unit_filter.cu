// Filter spectrum (call 1), spectrum layout conversion, diagnostics.
#include "hnd_kernels.cuh"
#include "hnd_multi2.cuh"
#include "hnd_filter2.cuh"
#include "hnd_kgrad.cuh"
#include "hnd_long1d.cuh"
#include "hnd_launch.h"
#include "hnd_host_util.h"

namespace hnd {

static SpecDims make_dims(int ndim, const int* n) {
  SpecDims d;
  d.ndim = ndim;
  for (int a = 0; a < 3; ++a) d.n[a] = a < ndim ? n[a] : 1;
  return d;
}

static unsigned grid_for(long long work, int threads) {
  long long b = (work + threads - 1) / threads;
  if (b < 1) b = 1;
  if (b > 148LL * 32) b = 148LL * 32;
  return static_cast<unsigned>(b);
}

// Zero the slots of `ngrids` grids [P0][P1][P2] with index P_a / 2 on some
// used axis a (the planes no kernel offset t in [-(n_a - 1), n_a - 1] is
// wrap-placed on); a slot on two such planes is written twice, with zero.
static __global__ void k_filter_clear_unmapped(float2* __restrict__ grid, int ndim, long long P0, long long P1,
                                               long long P2, long long plane_pts, long long ngrids) {
  const long long gsz = P0 * P1 * P2;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < plane_pts * ngrids;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long gi = e / plane_pts;
    long long r = e % plane_pts;
    long long s0, s1, s2;
    if (r < P1 * P2) {                               // axis 0 at P0 / 2
      s0 = P0 / 2, s1 = r / P2, s2 = r % P2;
    } else if (ndim > 1 && (r -= P1 * P2) < P0 * P2) {   // axis 1 at P1 / 2
      s0 = r / P2, s1 = P1 / 2, s2 = r % P2;
    } else {                                          // axis 2 at P2 / 2
      if (ndim > 1) r -= P0 * P2;
      s0 = r / P1, s1 = r % P1, s2 = P2 / 2;
    }
    *HND_G(&grid[gi * gsz + (s0 * P1 + s1) * P2 + s2]) = make_float2(0.f, 0.f);
  }
}

// 3D: natural spectrum or the filter's full grids -> library order
static cudaError_t spec3_in_go(const float2* src, float4* out, const int* n, long long C, long long pitch, float scale,
                               int pair, cudaStream_t st) {
  const size_t sm = hnd2::spec3_in_smem(n[0]);
  cudaError_t e = ensure_smem(hnd2::k_spec3_in, sm);
  if (e != cudaSuccess) return e;
  const long long nkb = (n[2] + 1 + hnd2::kS3 - 1) / hnd2::kS3;
  const long long grids = pair ? (C + 1) / 2 : C;      // a pair grid's CTAs write both channels
  const long long ctas = grids * 2LL * n[1] * nkb;
  if (ctas > 0x7fffffffLL) return cudaErrorInvalidValue;
  hnd2::k_spec3_in<<<static_cast<unsigned>(ctas), 256, sm, st>>>(src, out, n[0], n[1], n[2], C, pitch, scale, pair);
  return cudaGetLastError();
}

template <int HP, bool TAB>
static cudaError_t filter_mlp_go_t(const hnd2::FilterMlpArgs& fa, long long noff, cudaStream_t st) {
  auto kern = hnd2::k_filter_mlp2<HP, TAB>;
  cudaError_t e = ensure_smem(kern, hnd2::FilterSmem<HP>::bytes(96, TAB));     // the largest feature count
  if (e != cudaSuccess) return e;
  const long long blocks = (noff + hnd2::kFO - 1) / hnd2::kFO;
  // small offset grids: split the channels over a second grid dimension so
  // that about four CTAs per SM are in flight (each recomputes its hidden tile)
  hnd2::FilterMlpArgs g = fa;
  const int tiles = (fa.nc + hnd2::kFC - 1) / hnd2::kFC;
  long long groups = (4LL * sm_count() + blocks - 1) / blocks;
  if (groups > tiles) groups = tiles;
  if (groups < 1) groups = 1;
  const int per = static_cast<int>((tiles + groups - 1) / groups);
  g.cgroup = per * hnd2::kFC;
  const unsigned gy = static_cast<unsigned>((fa.nc + g.cgroup - 1) / g.cgroup);
  kern<<<dim3(static_cast<unsigned>(blocks), gy), hnd2::kFT, hnd2::FilterSmem<HP>::bytes(fa.fin, TAB), st>>>(g);
  return cudaGetLastError();
}

template <int HP>
static cudaError_t filter_mlp_go(const hnd2::FilterMlpArgs& fa, long long noff, cudaStream_t st) {
  return fa.tab ? filter_mlp_go_t<HP, true>(fa, noff, st) : filter_mlp_go_t<HP, false>(fa, noff, st);
}

long long filter_table_bytes(int hidden, int ndim, const int* n) {
  for (int a = 0; a < ndim; ++a)
    if (n[a] > 256) return 0;              // long 1D: the feature path (a table would be as large as the grid)
  const int HP = (hidden + 31) / 32 * 32;
  return hnd2::filter_table_floats(HP, ndim, n) * 4;
}

cudaError_t launch_filter_tables(const FilterLaunch& f, int ndim, const int* n, float* tab, cudaStream_t st) {
  const int HP = (f.hidden + 31) / 32 * 32;
  const long long cnt = hnd2::filter_trig_offset(HP, ndim, n);
  hnd2::k_filter_tables<<<grid_for(cnt, 256), 256, 0, st>>>(f.W1, f.hidden, HP, f.num_freqs, ndim, n[0],
                                                            ndim > 1 ? n[1] : 1, ndim > 2 ? n[2] : 1, tab);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? launch_filter_trig(f, ndim, n, tab, st) : e;
}

cudaError_t launch_filter_trig(const FilterLaunch& f, int ndim, const int* n, float* tab, cudaStream_t st) {
  const int HP = (f.hidden + 31) / 32 * 32;
  const long long cnt = static_cast<long long>(HP) * (2 * n[ndim - 1] - 1);
  hnd2::k_filter_trig<<<grid_for(cnt, 256), 256, 0, st>>>(tab, HP, f.hidden, ndim, n[0], ndim > 1 ? n[1] : 1,
                                                          ndim > 2 ? n[2] : 1, f.gamma);
  return cudaGetLastError();
}

// Full transform of length 2N along one axis of the filter grid.
template <int N>
static cudaError_t fft_axis_go(float2* grid, const hnd2::AxisMap& m, cudaStream_t st) {
  auto kern = hnd2::k_fft_axis2<N>;
  const size_t sm = hnd2::AxisSmem<N>::kBytes;
  cudaError_t e = ensure_smem(kern, sm);
  if (e != cudaSuccess) return e;
  const long long per_cta = (hnd2::kAT / 32) * (32 / hnd2::P2<N>::G);
  long long blocks = (m.npencil + per_cta - 1) / per_cta;
  if (blocks > 148LL * 16) blocks = 148LL * 16;
  if (blocks < 1) blocks = 1;
  kern<<<static_cast<unsigned>(blocks), hnd2::kAT, sm, st>>>(grid, m);
  return cudaGetLastError();
}

static int lg2(long long x) {
  int l = 0;
  while ((1LL << l) < x) ++l;
  return l;
}

static cudaError_t fft_axis_n(int N, float2* grid, const hnd2::AxisMap& m, cudaStream_t st) {
  switch (N) {
    case 8: return fft_axis_go<8>(grid, m, st);
    case 16: return fft_axis_go<16>(grid, m, st);
    case 32: return fft_axis_go<32>(grid, m, st);
    case 64: return fft_axis_go<64>(grid, m, st);
    case 128: return fft_axis_go<128>(grid, m, st);
    case 256: return fft_axis_go<256>(grid, m, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_fft_axis(float2* grid, int ndim, const int* n, int axis, long long ngrids, cudaStream_t st) {
  long long gsz = 1, stride = 1;
  for (int a = 0; a < ndim; ++a) gsz *= 2 * n[a];
  for (int a = axis + 1; a < ndim; ++a) stride *= 2 * n[a];
  hnd2::AxisMap m;
  m.npencil = gsz * ngrids / (2 * n[axis]);
  m.lgS = m.lgSc = m.lgK = m.lgPi = lg2(stride);
  return fft_axis_n(n[axis], grid, m, st);
}

// ------------------------------------------------------------ long 1D
L1Split long1d_split(int n) {
  int lg = 0;
  while ((1LL << lg) < 2LL * n) ++lg;
  L1Split sp;
  sp.m = lg <= 18 ? 2 : 3;                 // factors of at most 2^9 points
  int left = lg;
  for (int a = 0; a < 3; ++a) {
    const int share = a < sp.m ? (left + (sp.m - a) - 1) / (sp.m - a) : 0;    // the larger shares first
    sp.P[a] = 1 << share;
    left -= share;
  }
  return sp;
}

// forward split transform on `ngrids` adjacent grids of P points
static cudaError_t l1_fwd(float2* grid, const L1Split& sp, long long ngrids, cudaStream_t st) {
  int h[3];
  long long P = 1;
  for (int a = 0; a < sp.m; ++a) {
    h[a] = sp.P[a] / 2;
    P *= sp.P[a];
  }
  long long Q = P;
  cudaError_t e = cudaSuccess;
  for (int a = 0; a < sp.m && e == cudaSuccess; ++a) {
    e = launch_fft_axis(grid, sp.m, h, a, ngrids, st);
    if (e != cudaSuccess || a == sp.m - 1) break;
    hnd2::k_l1_twiddle<<<grid_for(P * ngrids, 256), 256, 0, st>>>(grid, sp.P[a], Q, P * ngrids);
    e = cudaGetLastError();
    Q /= sp.P[a];
  }
  return e;
}

// on conjugated spectra in split order: the conjugate of the unnormalised
// inverse, in natural order
static cudaError_t l1_inv_conj(float2* grid, const L1Split& sp, long long ngrids, cudaStream_t st) {
  int h[3];
  long long P = 1;
  for (int a = 0; a < sp.m; ++a) {
    h[a] = sp.P[a] / 2;
    P *= sp.P[a];
  }
  cudaError_t e = cudaSuccess;
  for (int a = sp.m - 1; a >= 0 && e == cudaSuccess; --a) {
    e = launch_fft_axis(grid, sp.m, h, a, ngrids, st);
    if (e != cudaSuccess || a == 0) break;
    long long Q = 1;               // points of levels a - 1 .. m - 1
    for (int b = a - 1; b < sp.m; ++b) Q *= sp.P[b];
    hnd2::k_l1_twiddle<<<grid_for(P * ngrids, 256), 256, 0, st>>>(grid, sp.P[a - 1], Q, P * ngrids);
    e = cudaGetLastError();
  }
  return e;
}

size_t spectrum_set_bytes(int ndim, const int* n, long long C) {
  if (ndim == 1 && n[0] > 256) {
    const L1Split sp = long1d_split(n[0]);
    return static_cast<size_t>(hnd2::l1_spec_of(sp.m, sp.P).per_pair()) * 16 * static_cast<size_t>((C + 1) / 2);
  }
  return static_cast<size_t>(spec_per_channel(make_dims(ndim, n))) * 8 * static_cast<size_t>(C);
}

cudaError_t launch_fft_axes(float2* grid, int ndim, const int* n, long long ngrids, cudaStream_t st,
                            bool skip_zero) {
  long long gsz = 1;
  for (int a = 0; a < ndim; ++a) gsz *= 2 * n[a];
  cudaError_t e = cudaSuccess;
  for (int a = 0; a < ndim && e == cudaSuccess; ++a) {
    long long stride = 1;
    for (int b = a + 1; b < ndim; ++b) stride *= 2 * n[b];
    hnd2::AxisMap m;
    m.lgS = lg2(stride);
    m.lgSc = m.lgK = m.lgPi = m.lgS;
    long long inner = stride;
    if (skip_zero && a + 1 < ndim) {
      // axes after a are still zero-padded: only s_b < n_b is non-zero there
      if (a + 2 == ndim) {
        inner = n[a + 1];
        m.lgSc = m.lgK = m.lgPi = lg2(inner);
      } else {
        inner = static_cast<long long>(n[a + 1]) * n[a + 2];
        m.lgSc = lg2(inner);
        m.lgK = lg2(n[a + 2]);
        m.lgPi = lg2(2LL * n[a + 2]);
      }
    }
    m.npencil = gsz / (2LL * n[a] * stride) * inner * ngrids;
    e = fft_axis_n(n[a], grid, m, st);
  }
  return e;
}

cudaError_t launch_filter_chunk(const FilterLaunch& f, int ndim, const int* n, int c0, int nc, float2* grid,
                                void* spectrum, cudaStream_t st) {
  const SpecDims d = make_dims(ndim, n);
  long long gsz = 1, noff = 1;
  for (int a = 0; a < ndim; ++a) {
    gsz *= 2 * n[a];
    noff *= 2 * n[a] - 1;
  }
  // 2D, 3D and long 1D: two channels per complex grid (the kernel values are real)
  const bool long1d = ndim == 1 && n[0] > 256;
  const int pair = ndim >= 2 || long1d ? 1 : 0;
  const int ngrids = pair ? (nc + 1) / 2 : nc;
  // the network writes every slot an offset maps to; only the slots at index
  // n_a on some axis stay (no offset lands there), so those are cleared
  long long pa[3] = {1, 1, 1};
  for (int ax = 0; ax < ndim; ++ax) pa[ax] = 2LL * n[ax];
  long long plane_pts = 0;
  for (int ax = 0; ax < ndim; ++ax) plane_pts += gsz / pa[ax];
  k_filter_clear_unmapped<<<grid_for(plane_pts * ngrids, 256), 256, 0, st>>>(grid, ndim, pa[0], pa[1], pa[2],
                                                                              plane_pts, ngrids);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  hnd2::FilterMlpArgs fa;
  fa.W1 = f.W1;
  fa.b1 = f.b1;
  fa.W2 = f.W2;
  fa.b2 = f.b2;
  fa.alpha = f.alpha;
  fa.num_freqs = f.num_freqs;
  fa.hidden = f.hidden;
  fa.fin = 2 * f.num_freqs * ndim;
  fa.decay_scale = f.decay_scale;
  fa.window = f.window;
  fa.circular = f.circular;
  fa.ndim = ndim;
  for (int a = 0; a < 3; ++a) fa.n[a] = a < ndim ? n[a] : 1;
  fa.c0 = c0;
  fa.nc = nc;
  fa.grid = grid;
  fa.gamma = f.gamma;
  fa.beta = f.beta;
  fa.tab = f.tab;
  fa.pair = pair;
  const int HP = (f.hidden + 31) / 32 * 32;
  e = HP <= 32 ? filter_mlp_go<32>(fa, noff, st)
      : HP <= 64 ? filter_mlp_go<64>(fa, noff, st)
      : HP <= 96 ? filter_mlp_go<96>(fa, noff, st)
                 : filter_mlp_go<128>(fa, noff, st);
  if (e != cudaSuccess) return e;
  if (long1d) {
    const L1Split sp = long1d_split(n[0]);
    if ((e = l1_fwd(grid, sp, ngrids, st)) != cudaSuccess) return e;
    const hnd2::L1Spec d1 = hnd2::l1_spec_of(sp.m, sp.P);
    hnd2::k_l1_pair_store<<<grid_for(d1.per_pair() * ngrids, 256), 256, 0, st>>>(
        grid, static_cast<float4*>(spectrum), d1, c0 / 2, ngrids, static_cast<float>(1.0 / static_cast<double>(gsz)));
    return cudaGetLastError();
  }
  e = launch_fft_axes(grid, ndim, n, ngrids, st);
  if (e != cudaSuccess) return e;
  const long long per = spec_per_channel(d);
  const float scale = static_cast<float>(1.0 / static_cast<double>(gsz));
  if (ndim == 2) {
    float4* out = static_cast<float4*>(spectrum) + static_cast<long long>(c0) * (per / 2);
    hnd2::k_spec_import_v2<<<grid_for(per / 2 * nc, 256), 256, 0, st>>>(grid, out, n[0], n[1], nc, 2LL * n[1],
                                                                        scale, pair);
  } else if (ndim == 3) {
    float4* out = static_cast<float4*>(spectrum) + static_cast<long long>(c0) * (per / 2);
    if ((e = spec3_in_go(grid, out, n, nc, 2LL * n[2], scale, pair, st)) != cudaSuccess) return e;
  } else {
    k_spec_pack<<<grid_for(per * nc, 256), 256, 0, st>>>(grid, static_cast<float2*>(spectrum), d, c0, nc, scale);
  }
  return cudaGetLastError();
}

template <class T>
static cudaError_t kgrad_chunk_t(const KgradLaunch& g, cudaStream_t st) {
  hnd2::KgDims d;
  d.n0 = g.n[0];
  d.n1 = g.ndim > 1 ? g.n[1] : 1;
  d.n2 = g.ndim > 2 ? g.n[2] : 1;
  d.P0 = 2 * d.n0;
  d.P1 = g.ndim > 1 ? 2 * d.n1 : 1;
  d.P2 = g.ndim > 2 ? 2 * d.n2 : 1;
  d.l0 = lg2(d.P0);
  d.l1 = lg2(d.P1);
  d.l2 = lg2(d.P2);
  const long long gsz = static_cast<long long>(d.P0) * d.P1 * d.P2;
  const int nvol = g.ncc * g.B;
  float2* gw = g.grids;
  float2* acc = gw + gsz * nvol;
  const int nh = (g.ncc + 1) / 2;
  hnd2::k_kg_pad<T><<<grid_for(gsz * nvol, 256), 256, 0, st>>>(
      static_cast<const T*>(g.k), static_cast<const T*>(g.v), static_cast<const T*>(g.q), static_cast<const T*>(g.dy),
      gw, d, g.B, g.C, g.c0, nvol);
  const bool long1d = g.ndim == 1 && g.n[0] > 256;
  const L1Split sp = long1d ? long1d_split(g.n[0]) : L1Split();
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess)
    e = long1d ? l1_fwd(gw, sp, nvol, st) : launch_fft_axes(gw, g.ndim, g.n, nvol, st, true);
  if (e != cudaSuccess) return e;
  hnd2::k_kg_corr<<<grid_for(gsz * nh, 256), 256, 0, st>>>(gw, acc, d, g.B, g.ncc, gsz, long1d ? sp.P[0] : 0,
                                                             long1d ? sp.P[1] : 1, long1d ? sp.P[2] : 1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // acc holds conj(A_c1 + i A_c2): a forward transform gives the conjugate of
  // the unnormalised inverse, dK_c1 - i dK_c2
  e = long1d ? l1_inv_conj(acc, sp, nh, st) : launch_fft_axes(acc, g.ndim, g.n, nh, st);
  if (e != cudaSuccess) return e;
  const float scale = static_cast<float>(1.0 / static_cast<double>(gsz));
  if (g.circular) {
    const long long nper = static_cast<long long>(d.n0) * d.n1 * d.n2;
    hnd2::k_kg_extract_periodic<<<grid_for(nper * g.ncc, 256), 256, 0, st>>>(acc, g.dK, d, g.c0, g.ncc, scale);
  } else {
    long long noff = 1;
    for (int a = 0; a < g.ndim; ++a) noff *= 2 * g.n[a] - 1;
    hnd2::k_kg_extract<<<grid_for(noff * g.ncc, 256), 256, 0, st>>>(acc, g.dK, d, g.c0, g.ncc, scale);
  }
  return cudaGetLastError();
}

cudaError_t launch_kgrad_chunk(const KgradLaunch& g, cudaStream_t st) {
  return g.bf16 ? kgrad_chunk_t<__nv_bfloat16>(g, st) : kgrad_chunk_t<float>(g, st);
}

cudaError_t launch_spec_convert(int ndim, const int* n, long long C, const void* src, void* dst, bool to_natural,
                                cudaStream_t st) {
  if (ndim == 1 && n[0] > 256) {
    const L1Split sp = long1d_split(n[0]);
    const hnd2::L1Spec d1 = hnd2::l1_spec_of(sp.m, sp.P);
    if (to_natural)
      hnd2::k_l1_spec_export<<<grid_for((n[0] + 1LL) * C, 256), 256, 0, st>>>(
          static_cast<const float4*>(src), static_cast<float2*>(dst), n[0], d1, C);
    else
      hnd2::k_l1_spec_import<<<grid_for(d1.per_pair() * ((C + 1) / 2), 256), 256, 0, st>>>(
          static_cast<const float2*>(src), static_cast<float4*>(dst), n[0], d1, C, n[0] + 1LL);
    return cudaGetLastError();
  }
  const SpecDims d = make_dims(ndim, n);
  const long long total = spec_per_channel(d) * C;
  if (ndim == 3) {
    if (to_natural)
      hnd2::k_spec3_out<<<grid_for(total / 2, 256), 256, 0, st>>>(static_cast<const float4*>(src),
                                                                 static_cast<float2*>(dst), n[0], n[1], n[2], C);
    else
      return spec3_in_go(static_cast<const float2*>(src), static_cast<float4*>(dst), n, C, n[2] + 1, 1.0f, 0, st);
    return cudaGetLastError();
  }
  if (ndim == 2) {
    if (to_natural)
      hnd2::k_spec_export_v2<<<grid_for(total / 2, 256), 256, 0, st>>>(static_cast<const float4*>(src),
                                                                      static_cast<float2*>(dst), n[0], n[1], C);
    else
      hnd2::k_spec_import_v2<<<grid_for(total / 2, 256), 256, 0, st>>>(static_cast<const float2*>(src),
                                                                      static_cast<float4*>(dst), n[0], n[1], C,
                                                                      n[1] + 1, 1.0f);
    return cudaGetLastError();
  }
  if (to_natural)
    k_spec_export<<<grid_for(total, 256), 256, 0, st>>>(static_cast<const float2*>(src), static_cast<float2*>(dst), d, C);
  else
    k_spec_import<<<grid_for(total, 256), 256, 0, st>>>(static_cast<const float2*>(src), static_cast<float2*>(dst), d, C);
  return cudaGetLastError();
}

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    cached[dev] = v;
  }
  return cached[dev];
}

cudaError_t launch_bounded_wait(int* status, const int* flag, long long limit_cycles, cudaStream_t st) {
  const long long max_it = limit_cycles / 1000 + 16;
  k_bounded_wait<<<1, 32, 0, st>>>(status, flag, limit_cycles, max_it);
  return cudaGetLastError();
}

}  // namespace hnd
