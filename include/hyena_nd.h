/*
 * hyena_nd.h -- C ABI of the B200 (sm_100a) gated nD FFT long-convolution library.
 *
 * The operation (HyenaND pages):
 *   * autognosis blog "Native multi-dimensional subquadratic operators via
 *     input-dependent long convolutions", section "HyenaND", output equation
 *     y[i] = sum_j phi(x[j]) x[j] K[i - j]: a global convolution of a gated input
 *     with an implicitly parameterised kernel, evaluated through FFTs.
 *   * gist.science summary of arXiv 2607.19378, section "Methodologie": native
 *     N-dimensional grids L1 x ... x LN (no rasterisation), a kernel given by a
 *     sine-activated coordinate MLP times a window, and zero padding to twice
 *     the grid for the non-circular (linear) convolution; section
 *     "Implementation: nSubQ": forward FFT, spectral modulation, inverse FFT and
 *     output cropping fused in one kernel with intermediates kept on chip.
 *
 * In Hyena form, per batch b and channel c, with u = k (.) v:
 *     y[b,c,i] = q[b,c,i] * sum_{j in [0,n)^d} u[b,c,j] * K_c[i - j],   i in [0,n)^d,
 * where K_c is defined on every offset t in [-(n_a - 1), n_a - 1] per axis.
 *
 * Conventions shared by every call:
 *   * All device memory is owned by the caller; the library never allocates
 *     or frees.  Every call is asynchronous on the given CUDA stream
 *     (cudaStream_t passed as void*; NULL = legacy default stream) and
 *     performs no host synchronisation, except hyena_nd_device_status.
 *     Convolutions on the multi-pass and long 1D tiers with several waves
 *     run the waves round-robin on the caller's stream and up to two side
 *     streams the library creates per device on first use: they are forked
 *     from the caller's stream with an event and joined back to it before
 *     the call returns, so the call stays ordered on the caller's stream.
 *     Calls from several host threads serialise their enqueue on those side
 *     streams.
 *   * Argument errors are detected on the host before anything is launched
 *     and returned synchronously.  A failed launch returns HYENA_ND_ERR_CUDA.
 *     Errors detected on the device are written to a status word held in the
 *     first 16 bytes of the workspace and read by hyena_nd_device_status.
 *     The first 256 bytes of the workspace are its control area.
 *   * Activations q, k, v, y: contiguous [B, C, n_1, ..., n_d], last axis
 *     fastest, all of one dtype (fp32 or bf16; bf16 outputs are rounded to
 *     nearest even).  Arithmetic is fp32 throughout.
 *   * Every device pointer must be 16-byte aligned.
 *   * The spectrum is complex64 in an order private to this library: write it
 *     with hyena_nd_filter_spectrum or hyena_nd_spectrum_import and read it
 *     back with hyena_nd_spectrum_export.  It already carries the inverse
 *     transform's 1 / prod(P) scale (P_a = 2 n_a).
 */
#ifndef HYENA_ND_H_
#define HYENA_ND_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HYENA_ND_API __attribute__((visibility("default")))
#else
#define HYENA_ND_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HYENA_ND_OK = 0,
  HYENA_ND_ERR_INVALID_ARG = 1,        /* null pointer, bad rank, B or C < 1, ... */
  HYENA_ND_ERR_UNSUPPORTED = 2,        /* valid problem outside the supported sizes */
  HYENA_ND_ERR_MISALIGNED = 3,         /* a device pointer is not 16-byte aligned */
  HYENA_ND_ERR_WORKSPACE_TOO_SMALL = 4,
  HYENA_ND_ERR_CUDA = 5,               /* a CUDA runtime call or launch failed */
  HYENA_ND_ERR_DEVICE_TIMEOUT = 6,     /* a bounded device-side wait gave up */
  HYENA_ND_ERR_DEVICE_BOUNDS = 7       /* a checked build caught an out-of-range index */
} hyena_nd_status;

typedef enum { HYENA_ND_F32 = 0, HYENA_ND_BF16 = 1 } hyena_nd_dtype;

/* Problem descriptor.
 *   ndim     1, 2 or 3.
 *   n[a]     grid extent of axis a (a < ndim), a power of two in [8, 256];
 *            for ndim == 3 the two outer axes are limited to [8, 128]; for
 *            ndim == 1 any power of two in [8, 2^26] (long 1D context:
 *            n > 256 runs the padded length-2n transform as a split
 *            2n = P0 P1 (P2) into two or three passes of at most 512 points,
 *            in waves of volumes through the workspace).
 *   B, C     batch and channel counts (>= 1).
 *   io_dtype dtype of q, k, v and y.
 *   circular 0: zero-padded linear convolution.  1: circular (periodic)
 *            convolution y[i] = q[i] sum_j u[j] Kper[(i - j) mod n] (arXiv
 *            2607.19378 summary, "Methodologie", boundary handling: circular
 *            convolutions for periodic systems).  The filter call then
 *            evaluates the network at each offset's representative in
 *            [-n/2, n/2), which gives the periodic kernel on the linear
 *            offsets (t and t - n carry the same value); the convolution
 *            calls are unchanged, since for i, j in [0, n) the linear sum
 *            over K[i - j] is then the circular one.  It runs through the
 *            same 2n grid as the linear mode.  Other values:
 *            HYENA_ND_ERR_INVALID_ARG. */
typedef struct {
  int ndim;
  int64_t n[3];
  int64_t B, C;
  hyena_nd_dtype io_dtype;
  int circular;
} hyena_nd_problem;

/* Implicit filter (pages: coordinate MLP with sine activation times a window).
 * For every offset t in [-(n_a-1), n_a-1]^d:
 *   phi(t)  = [sin(pi m t_a / n_a), cos(pi m t_a / n_a)] for a < ndim, m = 1..num_freqs,
 *             ordered [axis][m][sin, cos]            (2 * num_freqs * ndim features)
 *   h       = sin(W1 phi + b1)                       (hidden units; with FiLM,
 *             sin(gamma (W1 phi + b1) + beta), see hyena_nd_filter_spectrum_film)
 *   K_c(t)  = ((W2 h + b2)_c) * exp(-alpha_c * ||t||_2 / decay_scale)
 * Device pointers, fp32, row-major: W1 [hidden, 2*num_freqs*ndim], b1 [hidden],
 * W2 [C, hidden], b2 [C], alpha [C].  Limits: 1 <= num_freqs <= 16,
 * 1 <= hidden <= 128, decay_scale > 0.  window 0: exp(-alpha_c |t|_2 / s);
 * window 1: the Gaussian window exp(-alpha_c (|t|_2 / s)^2) (arXiv 2607.19378
 * summary, "Methodologie", kernel synthesis: a learnable Gaussian window times
 * the coordinate network; alpha_c is its learnable width); other values:
 * HYENA_ND_ERR_UNSUPPORTED. */
typedef struct {
  int num_freqs;
  int hidden;
  const float *W1, *b1, *W2, *b2, *alpha;
  float decay_scale;
  int window;
} hyena_nd_filter;

/* Size in bytes of the spectrum buffer for `p`: C channels of
 * prod_{a<d-1} P_a * (P_d/2 + 1) complex64 values.  The long 1D tier
 * (n > 256) stores channel pairs instead: for channels 2j and 2j + 1 of the
 * split 2n = Po Pc (Pc the last factor of the split), the two complex64
 * values A = (K_a + K_b)/2 and D = (K_a - K_b)/2 at the (Po/2 + 1) Pc
 * frequencies whose first-level index is at most Po/2 (the rest follow by
 * Hermitian symmetry); a missing last channel (odd C) counts as zero.
 * 0 if `p` is invalid or unsupported. */
HYENA_ND_API size_t hyena_nd_spectrum_bytes(const hyena_nd_problem* p);

/* Workspace bytes needed by every call below for problem `p` (a pure
 * function of the descriptor, at least 256 bytes: the control area, then the
 * largest of the convolution's waves of intermediates (64 MiB in the 2D
 * and 3D multi-pass tiers, 48 MiB in the long 1D tier), one channel chunk of
 * the filter call's padded grids plus its first-layer tables (up to 2.25 GiB)
 * and one channel chunk of the kernel gradient's grids (about 256 MiB); each
 * at least one volume or channel).  hyena_nd_workspace_bytes_for gives each
 * call's own, smaller need.
 * 0 if `p` is invalid or unsupported.  The same workspace may be reused by
 * consecutive calls on one stream. */
HYENA_ND_API size_t hyena_nd_workspace_bytes(const hyena_nd_problem* p);

/* The calls that use a workspace, for hyena_nd_workspace_bytes_for. */
typedef enum {
  HYENA_ND_CALL_ALL = 0,          /* every call: hyena_nd_workspace_bytes(p) */
  HYENA_ND_CALL_CONV = 1,         /* hyena_nd_fftconv, _batched, _backward */
  HYENA_ND_CALL_FILTER = 2,       /* hyena_nd_filter_spectrum, _film */
  HYENA_ND_CALL_KERNEL_GRAD = 3   /* hyena_nd_kernel_grad */
} hyena_nd_call;

/* Workspace bytes that the calls of one kind need for problem `p` (a pure
 * function of the descriptor, at least 256 bytes for the control area): the
 * convolution calls need only their waves' intermediates (none on the
 * single-launch tiers), the filter calls a channel chunk of grids and
 * tables, the kernel gradient a chunk of its grids.  A caller that only runs
 * convolutions can hold this much instead of hyena_nd_workspace_bytes(p);
 * each call checks its own figure.  0 if `p` is invalid or unsupported or
 * `call` is not one of the values above.  (A deployment convenience of this
 * library; the pages only ask for a preallocated, deterministic workspace.) */
HYENA_ND_API size_t hyena_nd_workspace_bytes_for(const hyena_nd_problem* p, hyena_nd_call call);

/* Execution plan of a problem, as the calls below run it (host only, no
 * device work; a pure function of the descriptor). */
typedef enum {
  HYENA_ND_TIER_ROWS_1D = 0,   /* 1D, n <= 256: one fused row kernel */
  HYENA_ND_TIER_FUSED_2D = 1,  /* 2D, both axes <= 64: one persistent fused kernel */
  HYENA_ND_TIER_MULTI_2D = 2,  /* other 2D grids: rows, column units, rows, in waves */
  HYENA_ND_TIER_MULTI_3D = 3,  /* 3D grids: rows, (y, z) slabs, rows, in waves */
  HYENA_ND_TIER_LONG_1D = 4    /* 1D, n > 256: split transform passes, in waves */
} hyena_nd_tier;

typedef struct {
  hyena_nd_tier tier;
  int64_t wave;           /* volumes per wave of the multi-pass tiers (long 1D: channel-pair grids;
                             0 for single-launch tiers) */
  int64_t waves;          /* waves per convolution (1 for single-launch tiers) */
  int launches;           /* kernel launches per convolution */
  int split_levels;       /* long 1D: factors of the split 2n = P0 P1 (P2) (0 otherwise) */
  int split[3];           /* long 1D: the factors (1 where unused) */
  int filter_chunk;       /* channels per chunk of the filter call */
  int kgrad_chunk;        /* channels per chunk of the kernel gradient */
  size_t workspace_bytes; /* hyena_nd_workspace_bytes(p) */
  size_t spectrum_bytes;  /* hyena_nd_spectrum_bytes(p) */
  int streams;            /* multi-pass and long 1D tiers: streams running the waves round-robin (the
                             caller's and up to two side streams of the library, forked from and
                             joined back to it); else 1 */
} hyena_nd_plan_info;

/* Fill `out` with the plan of `p`.  Errors: HYENA_ND_ERR_INVALID_ARG (null or
 * invalid problem), HYENA_ND_ERR_UNSUPPORTED (valid but outside the sizes). */
HYENA_ND_API hyena_nd_status hyena_nd_plan_info_get(const hyena_nd_problem* p, hyena_nd_plan_info* out);

/* Clear the workspace control area (enqueues a 256-byte memset on
 * `stream`).  Call once on a fresh workspace before the first call that uses
 * it; `ws_bytes` must be at least 256. */
HYENA_ND_API hyena_nd_status hyena_nd_workspace_init(void* ws, size_t ws_bytes, void* cuda_stream);

/* Call 1: evaluate the implicit filter on the offset grid, place it on the
 * zero-padded periodic grid P^d (offset t at slot t mod P_a, slot n_a zero),
 * take its real-input DFT, scale by 1/prod(P) and store it in the library's
 * spectrum order.  `spectrum`: hyena_nd_spectrum_bytes(p) bytes, written.
 * Pages: blog sections "nSubQ" (parameter computation) and "Implementation
 * patterns" (neural parameterisation); arXiv summary "Methodologie". */
HYENA_ND_API hyena_nd_status hyena_nd_filter_spectrum(const hyena_nd_problem* p, const hyena_nd_filter* f,
                                         void* spectrum, void* ws, size_t ws_bytes,
                                         void* cuda_stream);

/* Call 1 per sample with FiLM conditioning: the pages make the kernel depend
 * on the whole input sample through a control z(x) that modulates the
 * coordinate network feature-wise (FiLM) (arXiv 2607.19378 summary,
 * "Methodologie", input-dependent kernels via registers and FiLM).  With the
 * modulation of sample b given as gamma[b], beta[b] (one value per hidden
 * unit), the hidden layer becomes
 *     h_b = sin(gamma[b] (.) (W1 phi + b1) + beta[b])
 * and sample b's spectrum is written at spectrum + b * spectrum_batch_stride
 * (bytes), in library order, ready for the batched and backward calls with
 * the same stride.  Mapping z(x) to (gamma, beta) is the caller's.
 *   gamma, beta  device fp32 [B, hidden], 4-byte aligned.
 *   spectrum_batch_stride  >= hyena_nd_spectrum_bytes(p), a multiple of 16.
 * Errors as hyena_nd_filter_spectrum; a stride below one spectrum is
 * HYENA_ND_ERR_INVALID_ARG. */
HYENA_ND_API hyena_nd_status hyena_nd_filter_spectrum_film(const hyena_nd_problem* p, const hyena_nd_filter* f,
                                              const float* gamma, const float* beta, void* spectrum,
                                              int64_t spectrum_batch_stride, void* ws, size_t ws_bytes,
                                              void* cuda_stream);

/* Call 2 (one volume): the gated linear convolution for one (b, c) pair.
 * `p->B` and `p->C` must both be 1; `spectrum_c` holds that channel's
 * spectrum.  Same semantics as the batched call. */
HYENA_ND_API hyena_nd_status hyena_nd_fftconv(const hyena_nd_problem* p, const void* q, const void* k,
                                 const void* v, const void* spectrum_c, void* y, void* ws,
                                 size_t ws_bytes, void* cuda_stream);

/* Call 3 (batched over B and C): for every (b, c),
 *   y[b,c] = q[b,c] (.) crop_n( IFFT_P( FFT_P(pad_P(k[b,c] (.) v[b,c])) (.) S[b,c] ) )
 * i.e. the linear convolution defined at the top of this header.
 * q, k, v: read; y: written (may not alias q, k or v); all [B, C, n...].
 * `spectrum`: C spectra laid out as hyena_nd_filter_spectrum writes them.
 * `spectrum_batch_stride`: 0 = one spectrum per channel shared by every b;
 * otherwise sample b uses spectrum + b * spectrum_batch_stride bytes (a
 * per-sample spectrum set, multiple of 16 bytes).
 * `ws`: hyena_nd_workspace_bytes(p) bytes of device scratch. */
HYENA_ND_API hyena_nd_status hyena_nd_fftconv_batched(const hyena_nd_problem* p, const void* q,
                                         const void* k, const void* v, const void* spectrum,
                                         int64_t spectrum_batch_stride, void* y, void* ws,
                                         size_t ws_bytes, void* cuda_stream);

/* Backward of call 3: the gradients of a loss L with respect to q, k and v,
 * given dy = dL/dy (all [B, C, n...] in the problem's dtype).  With
 * u = k (.) v and w = crop_n(K_c * u) as in the forward,
 *   dq = dy (.) w
 *   du[j] = sum_{i in [0,n)^d} q[i] dy[i] K_c[i - j]      (the adjoint convolution)
 *   dk = v (.) du,   dv = k (.) du.
 * The adjoint is the same padded FFT convolution with the conjugate spectrum:
 * for a real K_c on the 2n grid, the transform of K_c[-t] is conj(S).  The
 * forward intermediates are recomputed, not stored (blog "Native
 * multi-dimensional subquadratic operators via input-dependent long
 * convolutions", sections "勾配フローと数値安定性" (gradient flow and
 * numerical stability: recompute the forward FFT in the backward) and
 * "具体的な実装パターン(PyTorch)" (an autograd function that keeps only
 * the inputs and the kernel parameters)).  Arithmetic is fp32 as in the forward.
 * Runs two convolutions: dq, then the adjoint, whose last stage writes both
 * dk and dv (6 launches per wave on the multi-pass tiers).
 * q, k, v, dy: read.  dq, dk, dv: written; none may overlap another output or
 * an input.  `spectrum`, `spectrum_batch_stride`, `ws`: as in call 3.  The
 * gradient with respect to the filter is not computed here. */
HYENA_ND_API hyena_nd_status hyena_nd_fftconv_backward(const hyena_nd_problem* p, const void* q, const void* k,
                                          const void* v, const void* spectrum,
                                          int64_t spectrum_batch_stride, const void* dy, void* dq,
                                          void* dk, void* dv, void* ws, size_t ws_bytes,
                                          void* cuda_stream);

/* Gradient with respect to the kernel values, given dy = dL/dy of call 3:
 *   dK[c, t] = sum_b sum_{i in [0,n)^d} q[b,c,i] dy[b,c,i] u[b,c,i - t],  u = k (.) v,
 * for every offset t in [-(n_1-1), n_1-1] x ... (terms with i - t outside the
 * grid are absent): the cross-correlation of q (.) dy with u, summed over the
 * batch (blog "Native multi-dimensional subquadratic operators via
 * input-dependent long convolutions", gradient sections: dK by correlation).
 * Computed through zero-padded transforms on the 2n grid with fp32
 * arithmetic; the sum over b runs in a fixed order (deterministic).
 * q, k, v, dy: [B, C, n...] in the problem's dtype, read.  dK: float32
 * [C, 2n_1-1, ..., 2n_d-1] (index t + n - 1), written; it may not overlap an
 * input.  Circular problems: dK is the gradient with respect to the periodic
 * kernel, dKper[c, tau] = sum_b sum_i q dy[i] u[(i - tau) mod n], float32
 * [C, n_1, ..., n_d] (the linear offsets t = tau mod n summed).  The chain into the filter's parameters is the caller's (the filter
 * call is its forward).  `ws`: hyena_nd_workspace_bytes(p) bytes. */
HYENA_ND_API hyena_nd_status hyena_nd_kernel_grad(const hyena_nd_problem* p, const void* q, const void* k,
                                     const void* v, const void* dy, float* dK, void* ws, size_t ws_bytes,
                                     void* cuda_stream);

/* Same operation as hyena_nd_fftconv_batched, for callers that cannot
 * allocate device memory and so have no workspace to pass: for instance a
 * plugin whose interface carries only input and output buffers, or an
 * application that reserves all device memory at start-up and allows no
 * allocation afterwards.  (The HyenaND pages have no counterpart; this is a
 * deployment convenience of this library.)
 * Scratch: a fixed array inside the library's device image -- a 256-byte
 * control area (the status word) followed by HYENA_ND_STATIC_SCRATCH_BYTES
 * (16 MiB) of scratch -- held by every GPU that loads the library until the
 * process exits.  Nothing is allocated or freed by the call.
 *   * A problem whose single (b, c) volume needs more scratch than that
 *     (8 bytes per voxel in the multi-pass tiers, e.g. a 128 x 128 x 256
 *     volume; 16 bytes per token in the long 1D tier, i.e. n > 2^20) returns
 *     HYENA_ND_ERR_WORKSPACE_TOO_SMALL before anything is launched.  Every
 *     other supported shape runs, on the same tier as the workspace call.
 *   * The first call on a device looks up the array's device address once;
 *     make that first call before any stream capture.
 *   * Every call shares the array and it keeps the previous call's contents
 *     (each call writes what it reads, so nothing has to start at zero).
 *     Calls whose kernels overlap on one GPU race on it: serialise them.
 *   * Device-side errors (a bounded wait of the fused 2D kernel that gives
 *     up) go to the array's status word, which is zero when the library loads
 *     and stays set until hyena_nd_device_status(NULL, stream) reads and
 *     clears it on the current device.
 *   * hyena_nd_last_launch_count reports the call's kernel launches.
 * Other arguments and errors: as hyena_nd_fftconv_batched. */
#define HYENA_ND_STATIC_SCRATCH_BYTES (16u << 20)
HYENA_ND_API hyena_nd_status hyena_nd_fftconv_batched_static(const hyena_nd_problem* p, const void* q,
                                                             const void* k, const void* v,
                                                             const void* spectrum,
                                                             int64_t spectrum_batch_stride, void* y,
                                                             void* cuda_stream);

/* Convert between the library's spectrum order and the natural order
 * [C, P_1, ..., P_{d-1}, P_d/2 + 1] complex64 (scale included, i.e. the
 * natural array is DFT(wrap-placed K) / prod(P)).  The library-order buffer
 * holds hyena_nd_spectrum_bytes(p) bytes, the natural one
 * 8 C prod_{a<d} P_a (n_d + 1) bytes (the same number except for the long 1D
 * tier, whose library order is the channel-pair layout described at
 * hyena_nd_spectrum_bytes); both are device memory and may not overlap.  The
 * import takes the other half by Hermitian symmetry where the library order
 * keeps it. */
HYENA_ND_API hyena_nd_status hyena_nd_spectrum_export(const hyena_nd_problem* p, const void* spectrum,
                                         void* natural_c64, void* cuda_stream);
HYENA_ND_API hyena_nd_status hyena_nd_spectrum_import(const hyena_nd_problem* p, const void* natural_c64,
                                         void* spectrum, void* cuda_stream);

/* Synchronise `stream`, then read and clear the device status word in `ws`
 * (a workspace), or, with ws == NULL, the status word of the fixed array of
 * hyena_nd_fftconv_batched_static on the current device.
 * Returns HYENA_ND_OK, the recorded device error, or HYENA_ND_ERR_CUDA. */
HYENA_ND_API hyena_nd_status hyena_nd_device_status(void* ws, void* cuda_stream);

/* Test hook for bounded device waits: launches one CTA that waits on a flag
 * nothing will ever set, with an iteration and clock limit of about
 * `limit_us` microseconds, after which it records HYENA_ND_ERR_DEVICE_TIMEOUT
 * in the status word and returns.  It never traps and never hangs. */
HYENA_ND_API hyena_nd_status hyena_nd_debug_bounded_wait(void* ws, size_t ws_bytes, int limit_us,
                                            void* cuda_stream);

/* Human-readable name of a status code (static string). */
HYENA_ND_API const char* hyena_nd_status_string(hyena_nd_status s);

/* Number of kernels the most recent successful call to hyena_nd_fftconv,
 * hyena_nd_fftconv_batched, hyena_nd_fftconv_batched_static or
 * hyena_nd_fftconv_backward on this host thread enqueued. */
HYENA_ND_API int hyena_nd_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* HYENA_ND_H_ */
