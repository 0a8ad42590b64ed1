// hnd_api.cu -- the C ABI declared in include/hyena_nd.h: argument checks,
// workspace planning, tier selection and launch sequencing.  Every arithmetic
// step of the convolution runs in the kernels of hnd_kernels.cuh.
#include "hyena_nd.h"
#include "hnd_bounds.cuh"
#include "hnd_launch.h"

#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <mutex>

namespace hnd {
cudaError_t launch_fused2d_f32(const ConvArgs& a);
cudaError_t launch_fused2d_bf16(const ConvArgs& a);
}  // namespace hnd

namespace {

thread_local int g_last_launches = 0;

}  // namespace

namespace hnd {

long long balanced_wave(long long pairs, long long B, size_t per_pair, size_t budget, bool whole_channels) {
  long long w = static_cast<long long>(budget / per_pair);
  if (w < 1) w = 1;
  if (w > pairs) w = pairs;
  if (whole_channels && w >= B) w -= w % B;        // keep a channel's samples in one wave
  // equal waves: no short last wave
  const long long nw = (pairs + w - 1) / w;
  long long we = (pairs + nw - 1) / nw;
  if (whole_channels && we >= B && we % B) we += B - we % B;
  return we < w ? we : w;
}

void note_launches(int n) { g_last_launches = n; }

cudaError_t side_stream(SideStream** out) {
  static std::mutex mu;
  static SideStream* per_dev[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(mu);
  if (!per_dev[dev]) {
    SideStream* r = new SideStream;
    for (int j = 1; j < SideStream::kMax; ++j)
      if ((e = cudaStreamCreateWithFlags(&r->s[j], cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&r->fork, cudaEventDisableTiming)) != cudaSuccess) return e;
    for (int j = 0; j < SideStream::kMax; ++j) {
      if ((e = cudaEventCreateWithFlags(&r->stagger[j], cudaEventDisableTiming)) != cudaSuccess) return e;
      if ((e = cudaEventCreateWithFlags(&r->join[j], cudaEventDisableTiming)) != cudaSuccess) return e;
    }
    per_dev[dev] = r;
  }
  *out = per_dev[dev];
  return cudaSuccess;
}

#ifdef HYENA_ND_BOUNDS
__device__ BoundsTable g_bounds;
__device__ __align__(16) unsigned char g_bounds_dummy[256];

cudaError_t bounds_register(const BoundsList& l, int* status, cudaStream_t st) {
  BoundsTable t{};
  for (int i = 0; i < l.n; ++i) {
    t.base[i] = reinterpret_cast<unsigned long long>(l.ptr[i]);
    t.bytes[i] = l.bytes[i];
  }
  t.n = l.n;
  t.status = status;
  return cudaMemcpyToSymbolAsync(g_bounds, &t, sizeof(t), 0, cudaMemcpyHostToDevice, st);
}
#else
cudaError_t bounds_register(const BoundsList&, int*, cudaStream_t) { return cudaSuccess; }
#endif

}  // namespace hnd

namespace {

constexpr size_t kStatusBytes = 256;                  // status word + padding
#ifndef HND_WAVE_MB
#define HND_WAVE_MB 64
#endif
#ifndef HND_STREAMS
#define HND_STREAMS 3
#endif
// Multi-pass tiers: intermediates of the waves in flight, split over
// HND_STREAMS streams that run the waves round-robin, each one stage behind
// the previous.  Measured on the 256^2, 64^3 and 128^3 grids: three streams
// with 64 MiB in all beat one stream with 96 MiB by 5%, 5% and 7%, and two
// or four streams, or larger budgets, by up to 4%.
constexpr size_t kWaveBudget = size_t(HND_WAVE_MB) << 20;
constexpr int kWaveStreams = HND_STREAMS;
static_assert(kWaveStreams >= 1 && kWaveStreams <= hnd::SideStream::kMax, "streams per convolution");
#ifndef HND_FILTER_MB
#define HND_FILTER_MB 2304
#endif
#ifndef HND_FILTER_MAXC
#define HND_FILTER_MAXC 128
#endif
// filter grids per channel chunk: each chunk evaluates the hidden layer once
// per offset, so fewer, larger chunks save that work at the cost of workspace
// (3D 128^3, C = 32: 28.0 / 18.7 / 14.7 ms per call at 256 / 512 / 1024 MiB
// before the later filter changes; 2.25 GiB holds all 32 channels of that
// grid in one chunk; only the filter call needs this workspace)
constexpr size_t kFilterBudget = size_t(HND_FILTER_MB) << 20;
constexpr int kFilterMaxChunk = HND_FILTER_MAXC;
constexpr size_t kKgradBudget = size_t(256) << 20;    // kernel-gradient grids per channel chunk
#ifndef HND_L1_WAVE_MB
#define HND_L1_WAVE_MB 48
#endif
// long 1D grids in flight: with several waves, three streams of 16 MiB each,
// so that a wave's grid stays in L2 across its passes (measured on 2^20
// tokens, C = 64: 1.96 ms against 2.09 with 3 x 32 MiB and 2.24 with one
// stream of 96 MiB)
constexpr size_t kL1WaveBudget = size_t(HND_L1_WAVE_MB) << 20;

enum Tier { kRows1D = 0, kFused2D = 1, kMulti2D = 2, kMulti3D = 3, kLong1D = 4 };

constexpr long long kLong1DMax = 1LL << 26;   // three split levels of at most 512 points

struct Plan {
  int ndim = 0;
  int n[3] = {1, 1, 1};
  long long B = 0, C = 0;
  int bf16 = 0;
  int circular = 0;
  long long L = 1;          // voxels per volume
  long long gsz = 1;        // padded grid points per channel
  int tier = 0;
  long long wave = 0;       // pairs per wave (multi-pass tiers)
  int streams = 1;          // multi-pass tiers: streams running alternate waves
  size_t wave_bytes = 0;    // workspace of one wave (multi-pass tiers)
  int filter_chunk = 1;
  int kgrad_chunk = 1;      // channels per kernel-gradient chunk
  size_t ws_total = 0;      // the largest of the three below (hyena_nd_workspace_bytes)
  size_t ws_conv = 0;       // convolution calls (forward, batched, backward)
  size_t ws_filter = 0;     // filter calls
  size_t ws_kgrad = 0;      // kernel gradient
  size_t spec_bytes = 0;
  size_t nat_bytes = 0;     // natural-order half spectrum (export / import)
  size_t filter_grid_bytes = 0;   // filter call: chunk grids (the tables follow)
};

bool pow2_in(long long x, long long lo, long long hi) { return x >= lo && x <= hi && (x & (x - 1)) == 0; }

hyena_nd_status make_plan(const hyena_nd_problem* p, Plan* pl) {
  if (!p) return HYENA_ND_ERR_INVALID_ARG;
  if (p->ndim < 1 || p->ndim > 3) return HYENA_ND_ERR_INVALID_ARG;
  if (p->B < 1 || p->C < 1) return HYENA_ND_ERR_INVALID_ARG;
  if (p->io_dtype != HYENA_ND_F32 && p->io_dtype != HYENA_ND_BF16) return HYENA_ND_ERR_INVALID_ARG;
  for (int a = 0; a < p->ndim; ++a)
    if (p->n[a] < 1) return HYENA_ND_ERR_INVALID_ARG;
  if (p->circular != 0 && p->circular != 1) return HYENA_ND_ERR_INVALID_ARG;
  if (p->ndim == 1) {
    if (!pow2_in(p->n[0], 8, kLong1DMax)) return HYENA_ND_ERR_UNSUPPORTED;
  } else {
    for (int a = 0; a < p->ndim; ++a)
      if (!pow2_in(p->n[a], 8, 256)) return HYENA_ND_ERR_UNSUPPORTED;
  }
  if (p->ndim == 3 && (p->n[0] > 128 || p->n[1] > 128)) return HYENA_ND_ERR_UNSUPPORTED;
  if (p->B > INT_MAX / p->C) return HYENA_ND_ERR_UNSUPPORTED;
  pl->ndim = p->ndim;
  pl->B = p->B;
  pl->C = p->C;
  pl->bf16 = p->io_dtype == HYENA_ND_BF16;
  pl->circular = p->circular;
  pl->L = 1;
  pl->gsz = 1;
  for (int a = 0; a < 3; ++a) pl->n[a] = 1;
  for (int a = 0; a < p->ndim; ++a) {
    pl->n[a] = static_cast<int>(p->n[a]);
    pl->L *= p->n[a];
    pl->gsz *= 2 * p->n[a];
  }
  const int nl = pl->n[p->ndim - 1];
  pl->spec_bytes = hnd::spectrum_set_bytes(p->ndim, pl->n, p->C);
  pl->nat_bytes = static_cast<size_t>(pl->gsz / (2 * nl) * (nl + 1)) * 8 * static_cast<size_t>(p->C);

  const long long pairs = p->B * p->C;
  size_t ws_conv = 0;
  if (p->ndim == 1 && nl > 256) {
    pl->tier = kLong1D;
    // one complex grid per channel pair of a sample
    const size_t per_grid = static_cast<size_t>(8) * static_cast<size_t>(pl->gsz);
    const long long grids = p->B * ((p->C + 1) / 2);
    pl->wave = hnd::balanced_wave(grids, 1, per_grid, kL1WaveBudget, false);
    pl->streams = 1;
    if (kWaveStreams > 1 && pl->wave < grids && per_grid * kWaveStreams <= kL1WaveBudget) {
      // several waves of grids small enough to share the budget: alternate
      // streams, each wave in its share
      pl->wave = hnd::balanced_wave(grids, 1, per_grid, kL1WaveBudget / kWaveStreams, false);
      const long long waves = (grids + pl->wave - 1) / pl->wave;
      pl->streams = static_cast<int>(waves < kWaveStreams ? waves : kWaveStreams);
    }
    pl->wave_bytes = (per_grid * static_cast<size_t>(pl->wave) + 255) / 256 * 256;
    ws_conv = pl->wave_bytes * static_cast<size_t>(pl->streams);
  } else if (p->ndim == 1) {
    pl->tier = kRows1D;
  } else if (hnd::fused_2d(p->ndim, pl->n)) {
    pl->tier = kFused2D;
  } else {
    pl->tier = p->ndim == 2 ? kMulti2D : kMulti3D;
    const size_t per_pair = static_cast<size_t>(8) * static_cast<size_t>(pl->L);
    pl->wave = hnd::balanced_wave(pairs, p->B, per_pair, kWaveBudget, true);
    pl->streams = 1;
    if (kWaveStreams > 1 && pl->wave < pairs) {
      // several waves: run them on two streams, each wave in half the budget
      pl->wave = hnd::balanced_wave(pairs, p->B, per_pair, kWaveBudget / kWaveStreams, true);
      const long long waves = (pairs + pl->wave - 1) / pl->wave;
      pl->streams = static_cast<int>(waves < kWaveStreams ? waves : kWaveStreams);
    }
    pl->wave_bytes = (per_pair * static_cast<size_t>(pl->wave) + 255) / 256 * 256;
    ws_conv = pl->wave_bytes * static_cast<size_t>(pl->streams);
  }
  // filter call: two channels per complex grid (the kernel values are real),
  // so a channel costs half a grid; the short 1D rows keep one per channel
  const bool fpair = p->ndim >= 2 || pl->tier == kLong1D;
  long long chunk = static_cast<long long>(kFilterBudget / ((fpair ? 4 : 8) * static_cast<size_t>(pl->gsz)));
  if (chunk < 1) chunk = 1;
  if (chunk > kFilterMaxChunk) chunk = kFilterMaxChunk;
  if (fpair && chunk > 1) chunk -= chunk % 2;        // whole pairs per chunk
  if (chunk > p->C) chunk = p->C;
  pl->filter_chunk = static_cast<int>(chunk);
  // the chunk's grids, then the first-layer tables (for the largest hidden width)
  const long long fgrids = fpair ? (chunk + 1) / 2 : chunk;
  pl->filter_grid_bytes = (static_cast<size_t>(fgrids) * static_cast<size_t>(pl->gsz) * 8 + 255) / 256 * 256;
  const size_t ws_filter = pl->filter_grid_bytes + static_cast<size_t>(hnd::filter_table_bytes(128, pl->ndim, pl->n));
  // kernel gradient: per channel B transformed grids (u + i z per sample) and
  // half an accumulator (two channels share one), P^d complex each
  const size_t per_kg = (static_cast<size_t>(p->B) + 1) * static_cast<size_t>(pl->gsz) * 8;
  long long kgc = static_cast<long long>(kKgradBudget / per_kg);
  if (kgc < 1) kgc = 1;
  if (kgc > p->C) kgc = p->C;
  pl->kgrad_chunk = static_cast<int>(kgc);
  const size_t ws_kgrad = per_kg * static_cast<size_t>(kgc);
  size_t need = ws_conv > ws_filter ? ws_conv : ws_filter;
  if (ws_kgrad > need) need = ws_kgrad;
  pl->ws_total = kStatusBytes + need;
  pl->ws_conv = kStatusBytes + ws_conv;
  pl->ws_filter = kStatusBytes + ws_filter;
  pl->ws_kgrad = kStatusBytes + ws_kgrad;
  return HYENA_ND_OK;
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

bool overlaps(const void* a, const void* b, size_t bytes) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + bytes && y < x + bytes;
}

// [a, a + na) and [b, b + nb) share a byte
bool overlaps2(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

hyena_nd_status cuda_status(cudaError_t e) { return e == cudaSuccess ? HYENA_ND_OK : HYENA_ND_ERR_CUDA; }

// Bytes of spectrum a convolution call may read: one set, or B sets at a
// byte stride.
size_t spectrum_span(const Plan& pl, int64_t sbs) {
  return sbs > 0 ? static_cast<size_t>(pl.B - 1) * static_cast<size_t>(sbs) + pl.spec_bytes : pl.spec_bytes;
}

// One gated convolution y = q . (K * (k . v)) (or with the conjugate
// spectrum) on the plan's tier; adds the kernel launches to *launches.
cudaError_t run_conv(const Plan& pl, const hnd::ConvArgs& a, void* ws, int* launches) {
  cudaError_t e = cudaSuccess;
  if (pl.tier == kRows1D) {
    e = hnd::launch_rows1d(a);
    *launches += 1;
  } else if (pl.tier == kFused2D) {
    e = pl.bf16 ? hnd::launch_fused2d_bf16(a) : hnd::launch_fused2d_f32(a);
    *launches += 1;
  } else {
    // multi-pass tiers: waves of (b, c) volumes, or of channel-pair grids in
    // the long 1D tier
    char* zbase = static_cast<char*>(ws) + kStatusBytes;
    const bool l1 = pl.tier == kLong1D;
    const long long pairs = l1 ? pl.B * ((pl.C + 1) / 2) : pl.B * pl.C;
    const int nl = pl.n[pl.ndim - 1];
    const int rp_total = static_cast<int>(pl.L / nl / 2);
    hnd::SideStream* side = nullptr;
    std::unique_lock<std::mutex> lk;
    const int ns = pl.streams;
    if (ns > 1) {
      // Waves go round-robin over the caller's stream and ns - 1 side
      // streams; side stream j starts one stage after stream j - 1 (it waits
      // for that stream's first forward rows), so that the column stage of
      // one wave shares the SMs with the row stages of the next.  Each
      // stream owns one wave-sized slice of the workspace.
      if ((e = hnd::side_stream(&side)) != cudaSuccess) return e;
      lk = std::unique_lock<std::mutex>(side->mu);
      if ((e = cudaEventRecord(side->fork, a.stream)) != cudaSuccess) return e;
      for (int j = 1; j < ns && e == cudaSuccess; ++j) e = cudaStreamWaitEvent(side->s[j], side->fork, 0);
      if (e != cudaSuccess) return e;
    }
    auto stream_of = [&](int lane) { return lane == 0 ? a.stream : side->s[lane]; };
    int w = 0;
    for (long long ord0 = 0; ord0 < pairs && e == cudaSuccess; ord0 += pl.wave, ++w) {
      const int np = static_cast<int>(pairs - ord0 < pl.wave ? pairs - ord0 : pl.wave);
      const int lane = ns > 1 ? w % ns : 0;
      hnd::ConvArgs aw = a;
      aw.stream = ns > 1 ? stream_of(lane) : a.stream;
      float2* zt = reinterpret_cast<float2*>(zbase + static_cast<size_t>(lane) * pl.wave_bytes);
      if (l1) {
        e = hnd::launch_long1d_wave(aw, zt, ord0, np, 0, launches);
      } else {
        e = hnd::launch_rowfwd(aw, nl, zt, ord0, np, rp_total);
        *launches += 1;
      }
      if (e == cudaSuccess && ns > 1 && w + 1 < ns) {
        // the next stream's first wave starts after this one's first stage
        e = cudaEventRecord(side->stagger[lane], aw.stream);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(side->s[lane + 1], side->stagger[lane], 0);
      }
      if (l1) {
        if (e == cudaSuccess) e = hnd::launch_long1d_wave(aw, zt, ord0, np, 1, launches);
        continue;
      }
      if (e == cudaSuccess) e = pl.tier == kMulti2D ? hnd::launch_mid1(aw, zt, ord0, np) : hnd::launch_mid2(aw, zt, ord0, np);
      if (e == cudaSuccess) e = hnd::launch_rowinv(aw, nl, zt, ord0, np, rp_total);
      *launches += 2;
    }
    for (int j = 1; j < ns; ++j) {
      // join: the caller's stream waits for every side stream's last wave
      const cudaError_t e1 = cudaEventRecord(side->join[j], side->s[j]);
      const cudaError_t e2 = e1 == cudaSuccess ? cudaStreamWaitEvent(a.stream, side->join[j], 0) : e1;
      if (e == cudaSuccess) e = e2;
    }
  }
  return e;
}

}  // namespace

extern "C" {

size_t hyena_nd_spectrum_bytes(const hyena_nd_problem* p) {
  Plan pl;
  return make_plan(p, &pl) == HYENA_ND_OK ? pl.spec_bytes : 0;
}

size_t hyena_nd_workspace_bytes(const hyena_nd_problem* p) {
  Plan pl;
  return make_plan(p, &pl) == HYENA_ND_OK ? pl.ws_total : 0;
}

size_t hyena_nd_workspace_bytes_for(const hyena_nd_problem* p, hyena_nd_call call) {
  Plan pl;
  if (make_plan(p, &pl) != HYENA_ND_OK) return 0;
  switch (call) {
    case HYENA_ND_CALL_ALL: return pl.ws_total;
    case HYENA_ND_CALL_CONV: return pl.ws_conv;
    case HYENA_ND_CALL_FILTER: return pl.ws_filter;
    case HYENA_ND_CALL_KERNEL_GRAD: return pl.ws_kgrad;
  }
  return 0;
}

hyena_nd_status hyena_nd_plan_info_get(const hyena_nd_problem* p, hyena_nd_plan_info* out) {
  if (!out) return HYENA_ND_ERR_INVALID_ARG;
  Plan pl;
  const hyena_nd_status st = make_plan(p, &pl);
  if (st != HYENA_ND_OK) return st;
  hyena_nd_plan_info info{};
  info.tier = static_cast<hyena_nd_tier>(pl.tier);
  // wave items: (b, c) volumes, or channel-pair grids in the long 1D tier
  const long long vols = pl.tier == kLong1D ? pl.B * ((pl.C + 1) / 2) : pl.B * pl.C;
  info.wave = pl.tier == kRows1D || pl.tier == kFused2D ? 0 : pl.wave;
  info.waves = info.wave > 0 ? (vols + pl.wave - 1) / pl.wave : 1;
  info.split[0] = info.split[1] = info.split[2] = 1;
  if (pl.tier == kLong1D) {
    const hnd::L1Split sp = hnd::long1d_split(pl.n[0]);
    info.split_levels = sp.m;
    for (int a = 0; a < 3; ++a) info.split[a] = sp.P[a];
    info.launches = static_cast<int>(info.waves) * hnd::long1d_conv_launches(pl.n[0]);
  } else {
    info.launches = info.wave > 0 ? static_cast<int>(info.waves) * 3 : 1;
  }
  info.filter_chunk = pl.filter_chunk;
  info.kgrad_chunk = pl.kgrad_chunk;
  info.workspace_bytes = pl.ws_total;
  info.spectrum_bytes = pl.spec_bytes;
  info.streams = pl.streams;
  *out = info;
  return HYENA_ND_OK;
}

hyena_nd_status hyena_nd_workspace_init(void* ws, size_t ws_bytes, void* cuda_stream) {
  if (!ws) return HYENA_ND_ERR_INVALID_ARG;
  if (!aligned16(ws)) return HYENA_ND_ERR_MISALIGNED;
  if (ws_bytes < kStatusBytes) return HYENA_ND_ERR_WORKSPACE_TOO_SMALL;
  return cuda_status(cudaMemsetAsync(ws, 0, kStatusBytes, static_cast<cudaStream_t>(cuda_stream)));
}

hyena_nd_status hyena_nd_fftconv_batched(const hyena_nd_problem* p, const void* q, const void* k, const void* v,
                                         const void* spectrum, int64_t spectrum_batch_stride, void* y, void* ws,
                                         size_t ws_bytes, void* cuda_stream) {
  Plan pl;
  hyena_nd_status st = make_plan(p, &pl);
  if (st != HYENA_ND_OK) return st;
  if (!q || !k || !v || !spectrum || !y || !ws) return HYENA_ND_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(spectrum) || !aligned16(y) || !aligned16(ws))
    return HYENA_ND_ERR_MISALIGNED;
  if (spectrum_batch_stride < 0) return HYENA_ND_ERR_INVALID_ARG;
  if (spectrum_batch_stride % 16 != 0) return HYENA_ND_ERR_MISALIGNED;
  if (ws_bytes < pl.ws_conv) return HYENA_ND_ERR_WORKSPACE_TOO_SMALL;
  const size_t act_bytes = static_cast<size_t>(pl.B * pl.C * pl.L) * (pl.bf16 ? 2 : 4);
  if (overlaps(y, q, act_bytes) || overlaps(y, k, act_bytes) || overlaps(y, v, act_bytes))
    return HYENA_ND_ERR_INVALID_ARG;

  hnd::ConvArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.spec = spectrum;
  a.sbs = spectrum_batch_stride / 8;
  a.y = y;
  a.B = static_cast<int>(pl.B);
  a.C = static_cast<int>(pl.C);
  a.bf16 = pl.bf16;
  a.ndim = pl.ndim;
  for (int i = 0; i < 3; ++i) a.n[i] = pl.n[i];
  a.stream = static_cast<cudaStream_t>(cuda_stream);
  a.status = static_cast<int*>(ws);

  hnd::BoundsList bl;
  bl.add(q, act_bytes);
  bl.add(k, act_bytes);
  bl.add(v, act_bytes);
  bl.add(y, act_bytes);
  bl.add(spectrum, spectrum_span(pl, spectrum_batch_stride));
  bl.add(ws, ws_bytes);
  if (hnd::bounds_register(bl, a.status, a.stream) != cudaSuccess) return HYENA_ND_ERR_CUDA;
  int launches = 0;
  if (run_conv(pl, a, ws, &launches) != cudaSuccess) return HYENA_ND_ERR_CUDA;
  g_last_launches = launches;
  return HYENA_ND_OK;
}

hyena_nd_status hyena_nd_fftconv(const hyena_nd_problem* p, const void* q, const void* k, const void* v,
                                 const void* spectrum_c, void* y, void* ws, size_t ws_bytes, void* cuda_stream) {
  if (!p) return HYENA_ND_ERR_INVALID_ARG;
  if (p->B != 1 || p->C != 1) return HYENA_ND_ERR_INVALID_ARG;
  return hyena_nd_fftconv_batched(p, q, k, v, spectrum_c, 0, y, ws, ws_bytes, cuda_stream);
}

hyena_nd_status hyena_nd_fftconv_backward(const hyena_nd_problem* p, const void* q, const void* k, const void* v,
                                          const void* spectrum, int64_t spectrum_batch_stride, const void* dy,
                                          void* dq, void* dk, void* dv, void* ws, size_t ws_bytes,
                                          void* cuda_stream) {
  Plan pl;
  hyena_nd_status st = make_plan(p, &pl);
  if (st != HYENA_ND_OK) return st;
  if (!q || !k || !v || !spectrum || !dy || !dq || !dk || !dv || !ws) return HYENA_ND_ERR_INVALID_ARG;
  const void* ptrs[9] = {q, k, v, spectrum, dy, dq, dk, dv, ws};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return HYENA_ND_ERR_MISALIGNED;
  if (spectrum_batch_stride < 0) return HYENA_ND_ERR_INVALID_ARG;
  if (spectrum_batch_stride % 16 != 0) return HYENA_ND_ERR_MISALIGNED;
  if (ws_bytes < pl.ws_conv) return HYENA_ND_ERR_WORKSPACE_TOO_SMALL;
  const size_t act_bytes = static_cast<size_t>(pl.B * pl.C * pl.L) * (pl.bf16 ? 2 : 4);
  const void* outs[3] = {dq, dk, dv};
  const void* ins[4] = {q, k, v, dy};
  for (int i = 0; i < 3; ++i) {
    for (const void* in : ins)
      if (overlaps(outs[i], in, act_bytes)) return HYENA_ND_ERR_INVALID_ARG;
    for (int j = i + 1; j < 3; ++j)
      if (overlaps(outs[i], outs[j], act_bytes)) return HYENA_ND_ERR_INVALID_ARG;
  }
  hnd::ConvArgs a;
  a.spec = spectrum;
  a.sbs = spectrum_batch_stride / 8;
  a.B = static_cast<int>(pl.B);
  a.C = static_cast<int>(pl.C);
  a.bf16 = pl.bf16;
  a.ndim = pl.ndim;
  for (int i = 0; i < 3; ++i) a.n[i] = pl.n[i];
  a.stream = static_cast<cudaStream_t>(cuda_stream);
  a.status = static_cast<int*>(ws);
  hnd::BoundsList bl;
  for (const void* ptr : {q, k, v, dy, static_cast<const void*>(dq), static_cast<const void*>(dk),
                          static_cast<const void*>(dv)})
    bl.add(ptr, act_bytes);
  bl.add(spectrum, spectrum_span(pl, spectrum_batch_stride));
  bl.add(ws, ws_bytes);
  if (hnd::bounds_register(bl, a.status, a.stream) != cudaSuccess) return HYENA_ND_ERR_CUDA;
  int launches = 0;
  // dq = dy . (K * (k . v)): the forward with dy as the output gate
  a.q = dy, a.k = k, a.v = v, a.y = dq, a.sconj = 1.f;
  cudaError_t e = run_conv(pl, a, ws, &launches);
  // du = K (adjoint) applied to q . dy: the conjugate spectrum; one convolution
  // writes both gated outputs dk = v . du and dv = k . du
  a.k = q, a.v = dy, a.sconj = -1.f;
  a.q = v, a.y = dk;
  a.g2 = k, a.y2 = dv;
  if (e == cudaSuccess) e = run_conv(pl, a, ws, &launches);
  if (e != cudaSuccess) return HYENA_ND_ERR_CUDA;
  g_last_launches = launches;
  return HYENA_ND_OK;
}

hyena_nd_status hyena_nd_kernel_grad(const hyena_nd_problem* p, const void* q, const void* k, const void* v,
                                     const void* dy, float* dK, void* ws, size_t ws_bytes, void* cuda_stream) {
  Plan pl;
  hyena_nd_status st = make_plan(p, &pl);
  if (st != HYENA_ND_OK) return st;
  if (!q || !k || !v || !dy || !dK || !ws) return HYENA_ND_ERR_INVALID_ARG;
  const void* ptrs[6] = {q, k, v, dy, dK, ws};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return HYENA_ND_ERR_MISALIGNED;
  if (ws_bytes < pl.ws_kgrad) return HYENA_ND_ERR_WORKSPACE_TOO_SMALL;
  long long noff = 1;     // dK entries per channel: linear offsets, or the periodic grid
  for (int a = 0; a < pl.ndim; ++a) noff *= pl.circular ? pl.n[a] : 2 * pl.n[a] - 1;
  const size_t act_bytes = static_cast<size_t>(pl.B * pl.C * pl.L) * (pl.bf16 ? 2 : 4);
  const size_t dk_bytes = static_cast<size_t>(pl.C * noff) * 4;
  const void* ins[4] = {q, k, v, dy};
  for (const void* in : ins)
    if (overlaps2(dK, dk_bytes, in, act_bytes)) return HYENA_ND_ERR_INVALID_ARG;
  hnd::KgradLaunch g;
  g.q = q;
  g.k = k;
  g.v = v;
  g.dy = dy;
  g.dK = dK;
  g.grids = reinterpret_cast<float2*>(static_cast<char*>(ws) + kStatusBytes);
  g.ndim = pl.ndim;
  for (int i = 0; i < 3; ++i) g.n[i] = pl.n[i];
  g.B = static_cast<int>(pl.B);
  g.C = static_cast<int>(pl.C);
  g.bf16 = pl.bf16;
  g.circular = pl.circular;
  hnd::BoundsList bl;
  for (const void* in : ins) bl.add(in, act_bytes);
  bl.add(dK, dk_bytes);
  bl.add(ws, ws_bytes);
  if (hnd::bounds_register(bl, static_cast<int*>(ws), static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess)
    return HYENA_ND_ERR_CUDA;
  // 2D multi-pass grids (linear mode) run the row-pair stages, which need half
  // the chunk workspace of the full-grid route
  const bool stages = pl.tier == kMulti2D && !pl.circular;
  for (long long c0 = 0; c0 < pl.C; c0 += pl.kgrad_chunk) {
    g.c0 = static_cast<int>(c0);
    g.ncc = static_cast<int>(pl.C - c0 < pl.kgrad_chunk ? pl.C - c0 : pl.kgrad_chunk);
    const cudaError_t e = stages ? hnd::launch_kgrad2d_chunk(g, static_cast<cudaStream_t>(cuda_stream))
                                 : hnd::launch_kgrad_chunk(g, static_cast<cudaStream_t>(cuda_stream));
    if (e != cudaSuccess) return HYENA_ND_ERR_CUDA;
  }
  return HYENA_ND_OK;
}

// Argument checks shared by the filter calls; fills `fl` from `f`.
static hyena_nd_status filter_args(const hyena_nd_filter* f, hnd::FilterLaunch* fl) {
  if (!f || !f->W1 || !f->b1 || !f->W2 || !f->b2 || !f->alpha) return HYENA_ND_ERR_INVALID_ARG;
  if (f->window != 0 && f->window != 1) return HYENA_ND_ERR_UNSUPPORTED;
  if (f->num_freqs < 1 || f->num_freqs > 16 || f->hidden < 1 || f->hidden > 128) return HYENA_ND_ERR_UNSUPPORTED;
  if (!(f->decay_scale > 0.f) || !std::isfinite(f->decay_scale)) return HYENA_ND_ERR_INVALID_ARG;
  const void* wp[5] = {f->W1, f->b1, f->W2, f->b2, f->alpha};
  for (const void* w : wp)
    if (reinterpret_cast<uintptr_t>(w) & 3u) return HYENA_ND_ERR_MISALIGNED;
  fl->W1 = f->W1;
  fl->b1 = f->b1;
  fl->W2 = f->W2;
  fl->b2 = f->b2;
  fl->alpha = f->alpha;
  fl->num_freqs = f->num_freqs;
  fl->hidden = f->hidden;
  fl->decay_scale = f->decay_scale;
  fl->window = f->window;
  return HYENA_ND_OK;
}

// The buffers a filter call reads and writes (checked build only).
static cudaError_t filter_bounds(const Plan& pl, const hyena_nd_filter* f, const void* spectrum, size_t spec_span,
                                 const void* ws, size_t ws_bytes, const float* gamma, const float* beta,
                                 cudaStream_t st) {
  const size_t fin = static_cast<size_t>(2 * f->num_freqs * pl.ndim), H = static_cast<size_t>(f->hidden);
  const size_t C = static_cast<size_t>(pl.C);
  hnd::BoundsList bl;
  bl.add(f->W1, 4 * H * fin);
  bl.add(f->b1, 4 * H);
  bl.add(f->W2, 4 * C * H);
  bl.add(f->b2, 4 * C);
  bl.add(f->alpha, 4 * C);
  bl.add(gamma, 4 * H * static_cast<size_t>(pl.B));
  bl.add(beta, 4 * H * static_cast<size_t>(pl.B));
  bl.add(spectrum, spec_span);
  bl.add(ws, ws_bytes);
  return hnd::bounds_register(bl, static_cast<int*>(const_cast<void*>(ws)), st);
}

static cudaError_t filter_all_chunks(const Plan& pl, const hnd::FilterLaunch& fl, void* spectrum, void* ws,
                                     cudaStream_t st) {
  float2* grid = reinterpret_cast<float2*>(static_cast<char*>(ws) + kStatusBytes);
  for (long long c0 = 0; c0 < pl.C; c0 += pl.filter_chunk) {
    const int nc = static_cast<int>(pl.C - c0 < pl.filter_chunk ? pl.C - c0 : pl.filter_chunk);
    cudaError_t e = hnd::launch_filter_chunk(fl, pl.ndim, pl.n, static_cast<int>(c0), nc, grid, spectrum, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

hyena_nd_status hyena_nd_filter_spectrum(const hyena_nd_problem* p, const hyena_nd_filter* f, void* spectrum,
                                         void* ws, size_t ws_bytes, void* cuda_stream) {
  Plan pl;
  hyena_nd_status st = make_plan(p, &pl);
  if (st != HYENA_ND_OK) return st;
  hnd::FilterLaunch fl;
  if ((st = filter_args(f, &fl)) != HYENA_ND_OK) return st;
  if (!spectrum || !ws) return HYENA_ND_ERR_INVALID_ARG;
  if (!aligned16(spectrum) || !aligned16(ws)) return HYENA_ND_ERR_MISALIGNED;
  if (ws_bytes < pl.ws_filter) return HYENA_ND_ERR_WORKSPACE_TOO_SMALL;
  fl.circular = pl.circular;
  if (filter_bounds(pl, f, spectrum, pl.spec_bytes, ws, ws_bytes, nullptr, nullptr,
                    static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess)
    return HYENA_ND_ERR_CUDA;
  if (hnd::filter_table_bytes(fl.hidden, pl.ndim, pl.n) > 0) {
    float* tab = reinterpret_cast<float*>(static_cast<char*>(ws) + kStatusBytes + pl.filter_grid_bytes);
    if (hnd::launch_filter_tables(fl, pl.ndim, pl.n, tab, static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess)
      return HYENA_ND_ERR_CUDA;
    fl.tab = tab;
  }
  return cuda_status(filter_all_chunks(pl, fl, spectrum, ws, static_cast<cudaStream_t>(cuda_stream)));
}

hyena_nd_status hyena_nd_filter_spectrum_film(const hyena_nd_problem* p, const hyena_nd_filter* f,
                                              const float* gamma, const float* beta, void* spectrum,
                                              int64_t spectrum_batch_stride, void* ws, size_t ws_bytes,
                                              void* cuda_stream) {
  Plan pl;
  hyena_nd_status st = make_plan(p, &pl);
  if (st != HYENA_ND_OK) return st;
  hnd::FilterLaunch fl;
  if ((st = filter_args(f, &fl)) != HYENA_ND_OK) return st;
  if (!gamma || !beta || !spectrum || !ws) return HYENA_ND_ERR_INVALID_ARG;
  if (!aligned16(spectrum) || !aligned16(ws)) return HYENA_ND_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(gamma) & 3u) || (reinterpret_cast<uintptr_t>(beta) & 3u))
    return HYENA_ND_ERR_MISALIGNED;
  if (spectrum_batch_stride % 16 != 0) return HYENA_ND_ERR_MISALIGNED;
  if (spectrum_batch_stride < static_cast<int64_t>(pl.spec_bytes)) return HYENA_ND_ERR_INVALID_ARG;
  if (ws_bytes < pl.ws_filter) return HYENA_ND_ERR_WORKSPACE_TOO_SMALL;
  fl.circular = pl.circular;
  if (filter_bounds(pl, f, spectrum, static_cast<size_t>(pl.B - 1) * static_cast<size_t>(spectrum_batch_stride) +
                                         pl.spec_bytes,
                    ws, ws_bytes, gamma, beta, static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess)
    return HYENA_ND_ERR_CUDA;
  if (hnd::filter_table_bytes(fl.hidden, pl.ndim, pl.n) > 0) {
    float* tab = reinterpret_cast<float*>(static_cast<char*>(ws) + kStatusBytes + pl.filter_grid_bytes);
    if (hnd::launch_filter_tables(fl, pl.ndim, pl.n, tab, static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess)
      return HYENA_ND_ERR_CUDA;
    fl.tab = tab;
  }
  for (long long b = 0; b < pl.B; ++b) {
    fl.gamma = gamma + b * f->hidden;
    fl.beta = beta + b * f->hidden;
    void* sb = static_cast<char*>(spectrum) + b * spectrum_batch_stride;
    if (fl.tab && hnd::launch_filter_trig(fl, pl.ndim, pl.n, const_cast<float*>(fl.tab),
                                          static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess)
      return HYENA_ND_ERR_CUDA;
    cudaError_t e = filter_all_chunks(pl, fl, sb, ws, static_cast<cudaStream_t>(cuda_stream));
    if (e != cudaSuccess) return HYENA_ND_ERR_CUDA;
  }
  return HYENA_ND_OK;
}

static hyena_nd_status spec_convert(const hyena_nd_problem* p, const void* src, void* dst, bool to_natural,
                                    void* cuda_stream) {
  Plan pl;
  hyena_nd_status st = make_plan(p, &pl);
  if (st != HYENA_ND_OK) return st;
  if (!src || !dst) return HYENA_ND_ERR_INVALID_ARG;
  if (!aligned16(src) || !aligned16(dst)) return HYENA_ND_ERR_MISALIGNED;
  const size_t src_bytes = to_natural ? pl.spec_bytes : pl.nat_bytes;
  const size_t dst_bytes = to_natural ? pl.nat_bytes : pl.spec_bytes;
  if (overlaps2(src, src_bytes, dst, dst_bytes)) return HYENA_ND_ERR_INVALID_ARG;
  hnd::BoundsList bl;
  bl.add(src, src_bytes);
  bl.add(dst, dst_bytes);
  if (hnd::bounds_register(bl, nullptr, static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess)
    return HYENA_ND_ERR_CUDA;
  return cuda_status(hnd::launch_spec_convert(pl.ndim, pl.n, pl.C, src, dst, to_natural,
                                              static_cast<cudaStream_t>(cuda_stream)));
}

hyena_nd_status hyena_nd_spectrum_export(const hyena_nd_problem* p, const void* spectrum, void* natural_c64,
                                         void* cuda_stream) {
  return spec_convert(p, spectrum, natural_c64, true, cuda_stream);
}

hyena_nd_status hyena_nd_spectrum_import(const hyena_nd_problem* p, const void* natural_c64, void* spectrum,
                                         void* cuda_stream) {
  return spec_convert(p, natural_c64, spectrum, false, cuda_stream);
}

hyena_nd_status hyena_nd_device_status(void* ws, void* cuda_stream) {
  if (!ws) {
    // the status word of the fixed array of hyena_nd_fftconv_batched_static
    int* w = nullptr;
    if (hnd::static_status_word(&w) != cudaSuccess) return HYENA_ND_ERR_CUDA;
    ws = w;
  }
  if (!aligned16(ws)) return HYENA_ND_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return HYENA_ND_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return HYENA_ND_ERR_CUDA;
  if (v != 0 && cudaMemset(ws, 0, sizeof(int)) != cudaSuccess) return HYENA_ND_ERR_CUDA;
  if (v < 0 || v > HYENA_ND_ERR_DEVICE_BOUNDS) return HYENA_ND_ERR_CUDA;
  return static_cast<hyena_nd_status>(v);
}

hyena_nd_status hyena_nd_debug_bounded_wait(void* ws, size_t ws_bytes, int limit_us, void* cuda_stream) {
  if (!ws) return HYENA_ND_ERR_INVALID_ARG;
  if (!aligned16(ws)) return HYENA_ND_ERR_MISALIGNED;
  if (ws_bytes < kStatusBytes) return HYENA_ND_ERR_WORKSPACE_TOO_SMALL;
  if (limit_us < 1 || limit_us > 1000000) return HYENA_ND_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  int* status = static_cast<int*>(ws);
  int* flag = status + 1;                       // never set by anyone
  if (cudaMemsetAsync(flag, 0, sizeof(int), s) != cudaSuccess) return HYENA_ND_ERR_CUDA;
  const long long limit_cycles = static_cast<long long>(limit_us) * 2000;   // about 2 GHz
  return cuda_status(hnd::launch_bounded_wait(status, flag, limit_cycles, s));
}

const char* hyena_nd_status_string(hyena_nd_status s) {
  switch (s) {
    case HYENA_ND_OK: return "HYENA_ND_OK";
    case HYENA_ND_ERR_INVALID_ARG: return "HYENA_ND_ERR_INVALID_ARG";
    case HYENA_ND_ERR_UNSUPPORTED: return "HYENA_ND_ERR_UNSUPPORTED";
    case HYENA_ND_ERR_MISALIGNED: return "HYENA_ND_ERR_MISALIGNED";
    case HYENA_ND_ERR_WORKSPACE_TOO_SMALL: return "HYENA_ND_ERR_WORKSPACE_TOO_SMALL";
    case HYENA_ND_ERR_CUDA: return "HYENA_ND_ERR_CUDA";
    case HYENA_ND_ERR_DEVICE_TIMEOUT: return "HYENA_ND_ERR_DEVICE_TIMEOUT";
    case HYENA_ND_ERR_DEVICE_BOUNDS: return "HYENA_ND_ERR_DEVICE_BOUNDS";
  }
  return "HYENA_ND_ERR_UNKNOWN";
}

int hyena_nd_last_launch_count(void) { return g_last_launches; }

}  // extern "C"
