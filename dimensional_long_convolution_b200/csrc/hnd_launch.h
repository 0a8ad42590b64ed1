// hnd_launch.h -- host-side launchers shared by the instantiation units and
// the C ABI (hnd_api.cu).  Each launcher switches on the runtime sizes and
// returns cudaErrorInvalidValue for a size it has no instantiation for.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <mutex>

namespace hnd {

struct ConvArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* spec;
  long long sbs;          // per-sample spectrum stride in complex elements (0 = shared)
  void* y;
  int B, C;
  int bf16;               // 0 = fp32 activations, 1 = bf16
  int n[3];
  int ndim;
  cudaStream_t stream;
  int* status = nullptr;  // device status word (may be null)
  float sconj = 1.f;      // -1: multiply by the conjugate spectrum (the adjoint convolution)
  const void* g2 = nullptr;  // optional second output y2 = g2 . conv (same layout as q and y)
  void* y2 = nullptr;
};

// 2D problems whose axes are both <= 64 run on the persistent fused kernel;
// larger 2D grids and every 3D grid run the multi-pass tier.  2D and 3D
// spectra use the packed order of the two-path FFT core.
inline bool fused_2d(int ndim, const int* n) { return ndim == 2 && n[0] <= 64 && n[1] <= 64; }

// Streaming multiprocessors of the current device (cached per device).
int sm_count();

// Volumes per wave of a multi-pass tier: as many as `budget` bytes of
// intermediates hold (per_pair bytes each, at least one), then evened out so
// that no wave is short; with whole_channels, a multiple of B where possible
// so that the B samples sharing a channel spectrum run in one wave.
long long balanced_wave(long long pairs, long long B, size_t per_pair, size_t budget, bool whole_channels);
// Side streams per device (created on first use, kept until exit; s[0] is
// unused: lane 0 is the caller's stream) with the events that fork them from,
// stagger them against each other and join them back to the caller's
// stream; `mu` serialises the enqueue of calls that use them.
struct SideStream {
  static constexpr int kMax = 4;
  cudaStream_t s[kMax] = {};
  cudaEvent_t fork = nullptr, stagger[kMax] = {}, join[kMax] = {};
  std::mutex mu;
};
cudaError_t side_stream(SideStream** out);
// Record the kernel count of the latest successful convolution call on this
// host thread (read by hyena_nd_last_launch_count).
void note_launches(int n);
// Device address of the status word at the head of the fixed array used by
// hyena_nd_fftconv_batched_static, on the current device (looked up once per
// device).
cudaError_t static_status_word(int** out);

// Maximum dynamic shared memory per CTA on sm_100 (227 KB).
constexpr size_t kMaxSmem = 232448;

// Fused tiers (one launch).
cudaError_t launch_fused2d(const ConvArgs& a);
cudaError_t launch_rows1d(const ConvArgs& a);
size_t fused2d_smem(int n0, int n1);

// Multi-pass tier, one wave of pairs [ord0, ord0 + np) in channel-major order.
cudaError_t launch_rowfwd(const ConvArgs& a, int nl, float2* zt, long long ord0, int np, int rp_total);
cudaError_t launch_rowinv(const ConvArgs& a, int nl, const float2* zt, long long ord0, int np, int rp_total);
cudaError_t launch_mid1(const ConvArgs& a, float2* zt, long long ord0, int np);
cudaError_t launch_mid2(const ConvArgs& a, float2* zt, long long ord0, int np);
// the 3D slab stage per conjugation sign (launch_mid2 picks one by sconj)
cudaError_t launch_mid2_fwd(const ConvArgs& a, float2* zt, long long ord0, int np);
cudaError_t launch_mid2_adj(const ConvArgs& a, float2* zt, long long ord0, int np);
size_t mid2_smem(int n0, int n1, bool* pair_variant);

// Filter spectrum and layout conversion.
struct FilterLaunch {
  const float *W1, *b1, *W2, *b2, *alpha;
  int num_freqs, hidden;
  float decay_scale;
  int window = 0;         // 0: exp(-alpha |t| / s), 1: exp(-alpha (|t| / s)^2)
  int circular = 0;       // 1: periodic representatives (circular mode)
  const float* gamma = nullptr;   // FiLM modulation of the sine layer ([hidden] each), or null
  const float* beta = nullptr;
  const float* tab = nullptr;     // per-axis first-layer tables (launch_filter_tables), or null
};
// Per-axis first-layer tables of the filter network (bytes; 0 where the
// feature path is used instead), and the launch that fills them.
long long filter_table_bytes(int hidden, int ndim, const int* n);
cudaError_t launch_filter_tables(const FilterLaunch& f, int ndim, const int* n, float* tab, cudaStream_t st);
// The sine and cosine tables of the last axis, scaled by f.gamma (FiLM) when
// set: launch_filter_tables fills them with f's gamma, and a per-sample
// gamma refills them with this before that sample's chunks.
cudaError_t launch_filter_trig(const FilterLaunch& f, int ndim, const int* n, float* tab, cudaStream_t st);
cudaError_t launch_filter_chunk(const FilterLaunch& f, int ndim, const int* n, int c0, int nc, float2* grid,
                                void* spectrum, cudaStream_t st);
cudaError_t launch_spec_convert(int ndim, const int* n, long long C, const void* src, void* dst, bool to_natural,
                                cudaStream_t st);
// In-place full forward transform along one axis of `ngrids` grids [P^d].
cudaError_t launch_fft_axis(float2* grid, int ndim, const int* n, int axis, long long ngrids, cudaStream_t st);
// Long 1D tier (n > 256): the split P = 2n = P0 P1 (P2) into m = 2 or 3
// factors of at most 512 points (unused factors 1), and one convolution over
// all volumes in waves of `wave` grids (3 + 2 (2m - 1) launches a wave).
struct L1Split {
  int m = 0;
  int P[3] = {1, 1, 1};
};
L1Split long1d_split(int n);
// Kernel launches of one convolution wave: 2m - 1.
int long1d_conv_launches(int n);
// Channels 2j and 2j + 1 of a sample share one complex grid; `wave` counts
// these channel-pair grids (B ceil(C/2) in all).
cudaError_t launch_long1d(const ConvArgs& a, float2* grid, long long wave, int* launches);
// One wave of `cnt` channel-pair grids from pair v0 on a.stream: part 0 the
// first pass, part 1 the remaining 2m - 2, part 2 all 2m - 1.
cudaError_t launch_long1d_wave(const ConvArgs& a, float2* grid, long long v0, long long cnt, int part,
                               int* launches);
// Bytes of one spectrum set in library order (C channels; long 1D: the pair
// layout of ceil(C/2) channel pairs).
size_t spectrum_set_bytes(int ndim, const int* n, long long C);
// In-place full forward transforms along every axis of `ngrids` complex grids
// [P^d] (P_a = 2 n_a), adjacent in memory.  skip_zero: the grids hold
// zero-padded data (zero wherever some s_a >= n_a), so the pencils of each
// pass that only see such zeros are skipped.
cudaError_t launch_fft_axes(float2* grid, int ndim, const int* n, long long ngrids, cudaStream_t st,
                            bool skip_zero = false);

// Kernel-value gradient for channels [c0, c0 + ncc) (all B samples of each).
struct KgradLaunch {
  const void *q, *k, *v, *dy;
  float* dK;              // [C][2n-1 ...]
  float2* grids;          // (2 B + 1) ncc grids of P^d complex
  int ndim, n[3], B, C, c0, ncc, bf16;
  int circular;           // 1: fold onto the periodic grid, dK [C][n ...]
};
cudaError_t launch_kgrad_chunk(const KgradLaunch& g, cudaStream_t st);
// The same on the 2D multi-pass tier (linear mode) through the row-pair and
// half-spectrum stages: `grids` holds 2 B ncc volumes of packed row spectra
// (8 n0 n1 bytes each) and ncc channel grids (16 n0 n1 bytes each).
cudaError_t launch_kgrad2d_chunk(const KgradLaunch& g, cudaStream_t st);
cudaError_t launch_bounded_wait(int* status, const int* flag, long long limit_cycles, cudaStream_t st);

}  // namespace hnd
