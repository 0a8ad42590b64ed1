"""Float64 CPU oracle for the gated nD long convolution -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  It shares no code with the CUDA library
(no kernels, tables, layouts or helpers); the only module both sides use is the
seeded input generator ``dimensional_long_convolution_b200.workloads``, which
holds none of the method's arithmetic.

What is computed (HyenaND pages):
  * "Native multi-dimensional subquadratic operators via input-dependent long
    convolutions" (autognosis blog), section "HyenaND", the output equation
    y[i] = sum_j phi(x[j]) * x[j] * K[i - j]: a global convolution of the gated
    input with an implicit kernel.  In the Hyena form used here the content gate
    phi(x) is the tensor k, x is v, and an output gate q multiplies the result:
        y[b,c,i] = q[b,c,i] * sum_{j in [0,n)^d} k[b,c,j] v[b,c,j] K_c[i - j],
    for every output index i in [0,n)^d.  q == 1 gives the blog's equation.
  * gist.science summary of arXiv 2607.19378, section "Methodologie", bullet on
    boundary handling: zero-padding the input to twice the grid before the FFT
    gives the non-circular (linear) convolution above; "Implementation: nSubQ":
    forward FFT -> spectral modulation -> inverse FFT -> output cropping.
  * Same summary, "Methodologie", kernel parameterisation: the kernel is a
    coordinate MLP with sine activation on continuous offsets, times a window.

Readings taken where the pages are silent (also listed in the design notes):
  1. Orientation is convolution K[i - j] (not correlation).
  2. Kernel support is every offset t in [-(n_a - 1), n_a - 1] on each axis;
     P_a = 2 n_a is then exactly enough, offset +-n_a maps to an unused slot
     that holds 0.
  3. Output window is [0, n)^d (crop after wrap placement).
  4. Fourier features: sin(pi m t_a / n_a), cos(pi m t_a / n_a), m = 1..M, in
     the order [axis][m][sin, cos]; MLP h = sin(W1 phi + b1), K = W2 h + b2;
     window exp(-alpha_c ||t||_2 / s).
  5. The spectrum carries the 1/prod(P) inverse-DFT scale.

Each routine below says which of these it follows.  Parity pins live in
tests/test_oracle.py.
"""
from __future__ import annotations

import itertools
from typing import Sequence, Tuple

import numpy as np


# ------------------------------------------------------------------ the filter
def offsets_grid(dims: Sequence[int]) -> np.ndarray:
    """All integer offsets t in [-(n_a-1), n_a-1]^d, shape [(2n_1-1)...(2n_d-1), d]
    (reading 2).  Row-major over the offset axes."""
    axes = [np.arange(-(n - 1), n, dtype=np.float64) for n in dims]
    mesh = np.meshgrid(*axes, indexing="ij")
    return np.stack([m.reshape(-1) for m in mesh], axis=-1)


def fourier_features(t: np.ndarray, dims: Sequence[int], num_freqs: int) -> np.ndarray:
    """phi(t): per axis a and frequency m = 1..M, [sin(pi m t_a/n_a), cos(pi m t_a/n_a)]
    in the order [axis][m][sin, cos] (reading 4).  t: [N, d] -> [N, 2 M d]."""
    cols = []
    for a, n in enumerate(dims):
        x = t[:, a] / float(n)
        for m in range(1, num_freqs + 1):
            cols.append(np.sin(np.pi * m * x))
            cols.append(np.cos(np.pi * m * x))
    return np.stack(cols, axis=-1)


def implicit_kernel(filt, dims: Sequence[int], channels=None, chunk: int = 1 << 18, window: int = 0,
                    film=None) -> np.ndarray:
    """K_c(t) for every channel c (or the listed ``channels``) and offset t
    (pages: coordinate MLP with sine activation times a window; reading 4).
    window 0: exp(-alpha_c ||t||_2 / s); window 1: the Gaussian window of the
    arXiv summary ("Methodologie", kernel synthesis: a learnable Gaussian
    window times the coordinate network), read as exp(-alpha_c (||t||_2 / s)^2)
    with alpha_c the learnable width.  ``film`` = (gamma, beta), one value per
    hidden unit: the per-sample feature-wise modulation of the sine layer,
    h = sin(gamma (W1 phi + b1) + beta) (reading 18; the pages condition the
    coordinate network on a per-sample control through FiLM).  Computed in
    float64 from the fp32 parameters, ``chunk`` offsets at a time to bound
    memory.  Returns [C, 2n_1-1, ..., 2n_d-1]; index t + (n - 1)."""
    t_all = offsets_grid(dims)
    W1 = filt.W1.astype(np.float64)
    b1 = filt.b1.astype(np.float64)
    sel = np.arange(filt.W2.shape[0]) if channels is None else np.asarray(channels)
    W2 = filt.W2.astype(np.float64)[sel]
    b2 = filt.b2.astype(np.float64)[sel]
    alpha = filt.alpha.astype(np.float64)[sel]
    K = np.empty((len(sel), t_all.shape[0]), dtype=np.float64)
    for s0 in range(0, t_all.shape[0], chunk):
        t = t_all[s0: s0 + chunk]
        phi = fourier_features(t, dims, filt.num_freqs)
        pre = phi @ W1.T + b1                            # [N, H]
        if film is not None:
            pre = film[0].astype(np.float64) * pre + film[1].astype(np.float64)
        h = np.sin(pre)
        mlp = h @ W2.T + b2                              # [N, C]
        r = np.sqrt(np.sum(t * t, axis=-1))              # ||t||_2
        rs = r / float(filt.decay_scale)
        win = np.exp(-np.outer(rs * rs if window == 1 else rs, alpha))
        K[:, s0: s0 + chunk] = (mlp * win).T
    return K.reshape((len(sel),) + tuple(2 * n - 1 for n in dims))


def periodic_rep(t: np.ndarray, n: int) -> np.ndarray:
    """The representative of t mod n in [-n/2, n/2): the offset the periodic
    (circular) mode evaluates the filter at."""
    return (t + n // 2) % n - n // 2


def implicit_kernel_periodic(filt, dims: Sequence[int], channels=None, window: int = 0) -> np.ndarray:
    """Circular mode (arXiv 2607.19378 summary, "Methodologie", boundary
    handling: circular convolutions for periodic systems): the kernel on the
    periodic grid, Kper[c, tau] for tau in [0, n)^d, is the filter evaluated at
    each tau's representative in [-n/2, n/2) per axis (reading: the window
    then decays with the periodic distance).  Returns [C, n_1, ..., n_d]."""
    d = len(dims)
    taus = np.stack(np.meshgrid(*[np.arange(n) for n in dims], indexing="ij"), axis=-1).reshape(-1, d)
    reps = np.stack([periodic_rep(taus[:, a], n) for a, n in enumerate(dims)], axis=-1)
    full = implicit_kernel(filt, dims, channels=channels, window=window)      # [C, 2n-1, ...]
    idx = tuple(reps[:, a] + n - 1 for a, n in enumerate(dims))
    out = full[(slice(None),) + idx]
    return out.reshape((out.shape[0],) + tuple(dims))


def periodize_to_offsets(Kper: np.ndarray, dims: Sequence[int]) -> np.ndarray:
    """K_lin[t] = Kper[t mod n] on the linear offsets t in [-(n-1), n-1]^d:
    for i, j in [0, n) the circular sum over Kper[(i - j) mod n] equals the
    linear sum over K_lin[i - j]."""
    idx = [np.arange(-(n - 1), n) % n for n in dims]
    return Kper[np.ix_(np.arange(Kper.shape[0]), *idx)]


def kernel_grad_periodic_direct(q, k, v, dy, dims) -> np.ndarray:
    """dKper[c, tau] = sum_b sum_i q dy[b,c,i] u[b,c,(i - tau) mod n]: the
    kernel gradient of the circular mode, from its definition (one tau at a
    time).  Returns [C, n...]."""
    z, u = q * dy, k * v
    d = len(dims)
    out = np.zeros((q.shape[1],) + tuple(dims))
    for tau in itertools.product(*[range(n) for n in dims]):
        us = np.roll(u, shift=tau, axis=tuple(range(2, 2 + d)))          # us[i] = u[(i - tau) mod n]
        out[(slice(None),) + tau] = np.sum(z * us, axis=(0,) + tuple(range(2, 2 + d)))
    return out


def wrap_place(K: np.ndarray, dims: Sequence[int]) -> np.ndarray:
    """Place K (offsets [-(n-1), n-1] per axis) on the padded periodic grid
    P_a = 2 n_a: offset t goes to slot t mod P_a; slot n_a stays 0 (reading 2)."""
    lead = K.shape[: K.ndim - len(dims)]
    P = tuple(2 * n for n in dims)
    out = np.zeros(lead + P, dtype=K.dtype)
    idx = []
    for n in dims:
        t = np.arange(-(n - 1), n)
        idx.append(np.mod(t, 2 * n))
    out[(Ellipsis,) + np.ix_(*idx)] = K
    return out


# ---------------------------------------------------------------- naive DFT
def dft_matrix(P: int) -> np.ndarray:
    """F_P[j, k] = exp(-2 pi i ((j k) mod P) / P), built in float64 with the
    product reduced mod P first so the angle stays exact."""
    j = np.arange(P, dtype=np.int64)
    jk = np.mod(np.outer(j, j), P).astype(np.float64)
    return np.exp(-2j * np.pi * jk / P)


def _apply_along(x: np.ndarray, M: np.ndarray, axis: int) -> np.ndarray:
    """out[..., k, ...] = sum_j M[k, j] x[..., j, ...] along ``axis``."""
    x = np.moveaxis(x, axis, -1)
    y = x @ M.T
    return np.moveaxis(y, -1, axis)


def spectrum_full(K: np.ndarray, dims: Sequence[int]) -> np.ndarray:
    """Full complex DFT over P^d of the wrap-placed kernel, times 1/prod(P)
    (reading 5).  K: [C, 2n-1, ...] -> [C, P_1, ..., P_d]."""
    d = len(dims)
    x = wrap_place(K.astype(np.complex128), dims)
    for a in range(d):
        x = _apply_along(x, dft_matrix(2 * dims[a]), x.ndim - d + a)
    return x / float(np.prod([2 * n for n in dims]))


def spectrum_half(K: np.ndarray, dims: Sequence[int]) -> np.ndarray:
    """Natural-order half spectrum [C, P_1, ..., P_{d-1}, P_d/2 + 1] (the kept
    half of a real-input transform along the last axis), 1/prod(P) included."""
    S = spectrum_full(K, dims)
    return S[..., : dims[-1] + 1]


def spectrum_at(K: np.ndarray, dims: Sequence[int], points: np.ndarray) -> np.ndarray:
    """The spectrum's definition at chosen frequencies only, for grids too long
    for a dense DFT matrix: S[c, k] = (1/prod(P)) sum_t K_c[t]
    exp(-2 pi i sum_a k_a (t_a mod P_a) / P_a) over every offset t (reading 5).
    points: [M, 1 + d] rows (c, k_1..k_d).  Returns [M] complex128.  O(prod(2n-1))
    per point; the phase index is reduced mod P_a first so the angle is exact."""
    d = len(dims)
    P = [2 * n for n in dims]
    tgrid = np.stack(np.meshgrid(*[np.arange(-(n - 1), n) for n in dims], indexing="ij"), axis=-1).reshape(-1, d)
    out = np.empty(points.shape[0], dtype=np.complex128)
    for r, p in enumerate(points):
        c = int(p[0])
        ph = np.zeros(tgrid.shape[0], dtype=np.float64)
        for a in range(d):
            ph += np.mod(int(p[1 + a]) * np.mod(tgrid[:, a], P[a]), P[a]) / P[a]
        out[r] = np.sum(K[c].reshape(-1) * np.exp(-2j * np.pi * ph)) / float(np.prod(P))
    return out


def full_from_half(Sh: np.ndarray, dims: Sequence[int]) -> np.ndarray:
    """Rebuild the full spectrum from the half by Hermitian symmetry
    S[-k] = conj(S[k]) of the transform of a real kernel."""
    d = len(dims)
    P = [2 * n for n in dims]
    out = np.zeros(Sh.shape[:-1] + (P[-1],), dtype=np.complex128)
    out[..., : dims[-1] + 1] = Sh
    for kl in range(dims[-1] + 1, P[-1]):
        src = Sh[..., P[-1] - kl]
        # negate the other frequency indices: k_a -> (-k_a) mod P_a
        for a in range(d - 1):
            ax = src.ndim - (d - 1) + a
            src = np.take(src, np.mod(-np.arange(P[a]), P[a]), axis=ax)
        out[..., kl] = np.conj(src)
    return out


# ------------------------------------------------------------ convolution O2
def conv_dft(q: np.ndarray, k: np.ndarray, v: np.ndarray, S_full: np.ndarray,
             dims: Sequence[int]) -> np.ndarray:
    """Linear convolution through zero-padded DFTs (pages: forward FFT ->
    spectral modulation -> inverse FFT -> crop; padding to twice the grid makes
    it non-circular).  The padded transform is applied with the P x n block of
    the DFT matrix (the zero rows contribute nothing), the inverse keeps only
    the n cropped outputs.  S_full: [C, P...] with 1/prod(P) folded in.
    q, k, v: [B, C, n...] float64.  Returns y float64 [B, C, n...]."""
    d = len(dims)
    u = (k * v).astype(np.complex128)
    x = u
    for a, n in enumerate(dims):
        F = dft_matrix(2 * n)[:, :n]                  # zero-padded forward
        x = _apply_along(x, F, 2 + a)
    x = x * S_full[None]
    for a, n in enumerate(dims):
        Finv = np.conj(dft_matrix(2 * n))[:n, :]       # crop to [0, n)
        x = _apply_along(x, Finv, 2 + a)
    return q * x.real


# ------------------------------------------------------------ convolution O1
def conv_direct(q: np.ndarray, k: np.ndarray, v: np.ndarray, K: np.ndarray,
                dims: Sequence[int]) -> np.ndarray:
    """The definition itself: y[b,c,i] = q[b,c,i] * sum_j u[b,c,j] K_c[i - j]
    with u = k v (blog, section "HyenaND", output equation).  O(L^2); tiny
    grids only.  K: [C, 2n-1, ...] with index t + (n - 1)."""
    d = len(dims)
    B, C = q.shape[:2]
    u = (k * v).reshape(B, C, -1)
    y = np.zeros((B, C) + tuple(dims), dtype=np.float64)
    jgrid = np.stack(np.meshgrid(*[np.arange(n) for n in dims], indexing="ij"), axis=-1).reshape(-1, d)
    Kf = K.reshape(C, -1)
    strides = np.array([int(np.prod([2 * m - 1 for m in dims[a + 1:]])) for a in range(d)], dtype=np.int64)
    for i in itertools.product(*[range(n) for n in dims]):
        off = (np.array(i)[None, :] - jgrid) + (np.array(dims) - 1)[None, :]
        flat = off @ strides
        y[(slice(None), slice(None)) + i] = np.einsum("bcj,cj->bc", u, Kf[:, flat])
    return q * y


def conv_direct_at(q: np.ndarray, k: np.ndarray, v: np.ndarray, K: np.ndarray,
                   dims: Sequence[int], points: np.ndarray) -> np.ndarray:
    """The definition evaluated only at chosen outputs.  points: [M, 2 + d] rows
    (b, c, i_1..i_d).  Returns [M] float64.  O(L) per point."""
    d = len(dims)
    jgrid = np.stack(np.meshgrid(*[np.arange(n) for n in dims], indexing="ij"), axis=-1).reshape(-1, d)
    strides = np.array([int(np.prod([2 * m - 1 for m in dims[a + 1:]])) for a in range(d)], dtype=np.int64)
    out = np.empty(points.shape[0], dtype=np.float64)
    for r, p in enumerate(points):
        b, c = int(p[0]), int(p[1])
        i = np.asarray(p[2:], dtype=np.int64)
        off = (i[None, :] - jgrid) + (np.array(dims) - 1)[None, :]
        kk = K[c].reshape(-1)[off @ strides]
        u = (k[b, c] * v[b, c]).reshape(-1)
        out[r] = q[(b, c) + tuple(i)] * float(np.dot(u, kk))
    return out


def conv_circular(q: np.ndarray, k: np.ndarray, v: np.ndarray, Kper: np.ndarray,
                  dims: Sequence[int]) -> np.ndarray:
    """Circular convolution on the unpadded periodic grid (the pages' periodic
    mode): y[i] = q[i] sum_j u[j] Kper[(i - j) mod n].  Kper: [C, n...]."""
    d = len(dims)
    u = (k * v).astype(np.complex128)
    Kh = Kper.astype(np.complex128)
    x = u
    for a, n in enumerate(dims):
        x = _apply_along(x, dft_matrix(n), 2 + a)
        Kh = _apply_along(Kh, dft_matrix(n), 1 + a)
    x = x * Kh[None]
    for a, n in enumerate(dims):
        x = _apply_along(x, np.conj(dft_matrix(n)) / n, 2 + a)
    return q * x.real


# ---------------------------------------------------------------- backward
# Gradients of L with respect to q, k, v for dy = dL/dy, from the definition
# above: y = q * w with w[i] = sum_j u[j] K[i - j] and u = k v, so
#   dq = dy * w,  du[j] = sum_i q[i] dy[i] K[i - j],  dk = v du,  dv = k du.
# (Blog "Native multi-dimensional subquadratic operators via input-dependent
# long convolutions", sections on gradient flow and the PyTorch autograd
# pattern: the backward recomputes the forward FFT convolution.)
def corr_direct(z: np.ndarray, K: np.ndarray, dims: Sequence[int]) -> np.ndarray:
    """The adjoint of the cropped linear convolution, written out:
    du[b,c,j] = sum_{i in [0,n)^d} z[b,c,i] K_c[i - j], j in [0,n)^d.
    O(L^2); tiny grids only.  K: [C, 2n-1, ...] with index t + (n - 1)."""
    d = len(dims)
    B, C = z.shape[:2]
    zf = z.reshape(B, C, -1)
    du = np.zeros((B, C) + tuple(dims), dtype=np.float64)
    igrid = np.stack(np.meshgrid(*[np.arange(n) for n in dims], indexing="ij"), axis=-1).reshape(-1, d)
    Kf = K.reshape(C, -1)
    strides = np.array([int(np.prod([2 * m - 1 for m in dims[a + 1:]])) for a in range(d)], dtype=np.int64)
    for j in itertools.product(*[range(n) for n in dims]):
        off = (igrid - np.array(j)[None, :]) + (np.array(dims) - 1)[None, :]
        du[(slice(None), slice(None)) + j] = np.einsum("bci,ci->bc", zf, Kf[:, off @ strides])
    return du


def corr_direct_at(z: np.ndarray, K: np.ndarray, dims: Sequence[int], points: np.ndarray) -> np.ndarray:
    """corr_direct at chosen outputs only.  points: [M, 2 + d] rows
    (b, c, j_1..j_d).  O(L) per point."""
    d = len(dims)
    igrid = np.stack(np.meshgrid(*[np.arange(n) for n in dims], indexing="ij"), axis=-1).reshape(-1, d)
    strides = np.array([int(np.prod([2 * m - 1 for m in dims[a + 1:]])) for a in range(d)], dtype=np.int64)
    out = np.empty(points.shape[0], dtype=np.float64)
    for r, p in enumerate(points):
        b, c = int(p[0]), int(p[1])
        j = np.asarray(p[2:], dtype=np.int64)
        off = (igrid - j[None, :]) + (np.array(dims) - 1)[None, :]
        out[r] = float(np.dot(z[b, c].reshape(-1), K[c].reshape(-1)[off @ strides]))
    return out


def corr_dft(z: np.ndarray, S_full: np.ndarray, dims: Sequence[int]) -> np.ndarray:
    """The adjoint through zero-padded DFTs: on the 2n grid the transform of
    K[-t] is conj(S) for a real K, so the adjoint is conv_dft's steps with the
    conjugate spectrum (and no output gate)."""
    x = z.astype(np.complex128)
    for a, n in enumerate(dims):
        x = _apply_along(x, dft_matrix(2 * n)[:, :n], 2 + a)
    x = x * np.conj(S_full)[None]
    for a, n in enumerate(dims):
        x = _apply_along(x, np.conj(dft_matrix(2 * n))[:n, :], 2 + a)
    return x.real


def backward_dft(q, k, v, dy, S_full, dims) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """(dq, dk, dv) through the DFT route (float64)."""
    w = conv_dft(np.ones_like(q), k, v, S_full, dims)
    du = corr_dft(q * dy, S_full, dims)
    return dy * w, v * du, k * du


def backward_direct(q, k, v, dy, K, dims) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """(dq, dk, dv) by direct sums (float64, tiny grids)."""
    w = conv_direct(np.ones_like(q), k, v, K, dims)
    du = corr_direct(q * dy, K, dims)
    return dy * w, v * du, k * du


# ------------------------------------------------------- kernel-value gradient
# dL/dK for L = sum dy y: y[i] = q[i] sum_j u[j] K[i - j] gives
#   dK[c, t] = sum_b sum_{i in [0,n)^d} q[b,c,i] dy[b,c,i] u[b,c,i - t]
# for every offset t in [-(n-1), n-1]^d (terms with i - t outside the grid
# are absent): the cross-correlation of z = q dy with u, summed over the
# batch (blog, gradient sections: dK by correlation).
def kernel_grad_direct(q, k, v, dy, dims) -> np.ndarray:
    """The definition, one offset at a time.  Returns [C, 2n-1, ...]."""
    d = len(dims)
    B, C = q.shape[:2]
    z, u = q * dy, k * v
    out = np.zeros((C,) + tuple(2 * n - 1 for n in dims))
    for t in itertools.product(*[range(-(n - 1), n) for n in dims]):
        zi = tuple(slice(max(0, ta), n + min(0, ta)) for ta, n in zip(t, dims))
        uj = tuple(slice(max(0, -ta), n - max(0, ta)) for ta, n in zip(t, dims))
        val = np.sum(z[(slice(None), slice(None)) + zi] * u[(slice(None), slice(None)) + uj],
                     axis=tuple(range(2, 2 + d)))
        out[(slice(None),) + tuple(ta + n - 1 for ta, n in zip(t, dims))] = val.sum(axis=0)
    return out


def kernel_grad_at(q, k, v, dy, dims, points: np.ndarray) -> np.ndarray:
    """kernel_grad_direct at chosen (c, t_1..t_d) rows only.  O(B L) each."""
    z, u = q * dy, k * v
    out = np.empty(points.shape[0])
    for r, p in enumerate(points):
        c, t = int(p[0]), [int(x) for x in p[1:]]
        zi = tuple(slice(max(0, ta), n + min(0, ta)) for ta, n in zip(t, dims))
        uj = tuple(slice(max(0, -ta), n - max(0, ta)) for ta, n in zip(t, dims))
        out[r] = float(np.sum(z[(slice(None), c) + zi] * u[(slice(None), c) + uj]))
    return out


def kernel_grad_dft(q, k, v, dy, dims) -> np.ndarray:
    """Through zero-padded DFTs: correlation = IDFT(sum_b Z_b conj(U_b)) on
    the 2n grid, read back at slot t mod 2n.  Returns [C, 2n-1, ...]."""
    d = len(dims)
    z, u = (q * dy).astype(np.complex128), (k * v).astype(np.complex128)
    for a, n in enumerate(dims):
        F = dft_matrix(2 * n)[:, :n]
        z = _apply_along(z, F, 2 + a)
        u = _apply_along(u, F, 2 + a)
    acc = np.sum(z * np.conj(u), axis=0)                  # [C, P...]
    for a, n in enumerate(dims):
        acc = _apply_along(acc, np.conj(dft_matrix(2 * n)) / (2 * n), 1 + a)
    idx = [np.arange(-(n - 1), n) % (2 * n) for n in dims]
    return acc.real[np.ix_(np.arange(acc.shape[0]), *idx)]


# -------------------------------------------------------------- conveniences
def reference_output(inputs, S_full=None, K=None) -> np.ndarray:
    """y for a seeded workload through O2 (float64)."""
    wl = inputs.wl
    if K is None:
        K = implicit_kernel(inputs.filt, wl.dims)
    if S_full is None:
        S_full = spectrum_full(K, wl.dims)
    return conv_dft(inputs.as_f64("q"), inputs.as_f64("k"), inputs.as_f64("v"), S_full, wl.dims)


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    """||a - b||_2 / ||b||_2 over all elements (complex values compared as
    complex numbers)."""
    cplx = np.iscomplexobj(a) or np.iscomplexobj(b)
    a = np.asarray(a, dtype=np.complex128 if cplx else np.float64)
    b = np.asarray(b, dtype=np.complex128 if cplx else np.float64)
    den = np.linalg.norm(b.reshape(-1))
    return float(np.linalg.norm((a - b).reshape(-1)) / (den if den > 0 else 1.0))
