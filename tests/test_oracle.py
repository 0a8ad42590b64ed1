"""Pins for the float64 oracle, each against something other than the oracle
itself: brute force, numpy library routines, closed forms and invariants of the
gated linear convolution y[i] = q[i] sum_j k[j] v[j] K[i - j]
(HyenaND blog, section "HyenaND", output equation; zero-padded linear mode from
the arXiv 2607.19378 summary, "Methodologie", boundary handling)."""
import itertools

import numpy as np
import pytest

from dimensional_long_convolution_b200 import workloads as W
from oracle import hyena_nd_oracle as O


def _rand_problem(dims, B=2, C=3, seed=0):
    rng = np.random.default_rng(seed)
    shape = (B, C) + tuple(dims)
    q, k, v = (rng.standard_normal(shape) for _ in range(3))
    K = rng.standard_normal((C,) + tuple(2 * n - 1 for n in dims))
    return q, k, v, K


# ---------------------------------------------------------------- brute force
@pytest.mark.parametrize("dims", [(8,), (5,), (6, 5), (4, 7), (8, 8), (3, 4, 5), (4, 4, 4)])
def test_dft_path_equals_direct_sum(dims):
    q, k, v, K = _rand_problem(dims)
    S = O.spectrum_full(K, dims)
    y2 = O.conv_dft(q, k, v, S, dims)
    y1 = O.conv_direct(q, k, v, K, dims)
    assert O.rel_l2(y2, y1) < 1e-12


def test_direct_sum_by_explicit_loops():
    """Fully scalar brute force of the definition on a tiny 2D grid."""
    dims = (3, 4)
    q, k, v, K = _rand_problem(dims, B=1, C=2, seed=3)
    y = O.conv_direct(q, k, v, K, dims)
    for c in range(2):
        for i0 in range(3):
            for i1 in range(4):
                s = 0.0
                for j0 in range(3):
                    for j1 in range(4):
                        s += k[0, c, j0, j1] * v[0, c, j0, j1] * K[c, i0 - j0 + 2, i1 - j1 + 3]
                assert abs(q[0, c, i0, i1] * s - y[0, c, i0, i1]) < 1e-12 * (1 + abs(s))


def test_direct_at_points_matches_full():
    dims = (6, 5)
    q, k, v, K = _rand_problem(dims, seed=5)
    y = O.conv_direct(q, k, v, K, dims)
    pts = np.array([[0, 0, 0, 0], [1, 2, 5, 4], [1, 1, 3, 2], [0, 2, 5, 0]])
    got = O.conv_direct_at(q, k, v, K, dims, pts)
    want = np.array([y[tuple(p)] for p in pts])
    assert np.max(np.abs(got - want)) < 1e-12


# ------------------------------------------------------- library special cases
@pytest.mark.parametrize("n", [8, 13, 32])
def test_1d_matches_numpy_convolve(n):
    rng = np.random.default_rng(n)
    u = rng.standard_normal(n)
    Kf = rng.standard_normal(2 * n - 1)              # offsets -(n-1)..(n-1)
    q = np.ones((1, 1, n))
    k = u.reshape(1, 1, n)
    v = np.ones((1, 1, n))
    S = O.spectrum_full(Kf.reshape(1, -1), (n,))
    y = O.conv_dft(q, k, v, S, (n,))[0, 0]
    want = np.convolve(u, Kf)[n - 1: 2 * n - 1]
    assert np.max(np.abs(y - want)) < 1e-12 * np.max(np.abs(want))


def test_separable_kernel_matches_sequential_1d_convolutions():
    n0, n1 = 6, 8
    rng = np.random.default_rng(11)
    u = rng.standard_normal((n0, n1))
    K0 = rng.standard_normal(2 * n0 - 1)
    K1 = rng.standard_normal(2 * n1 - 1)
    K = np.outer(K0, K1).reshape(1, 2 * n0 - 1, 2 * n1 - 1)
    S = O.spectrum_full(K, (n0, n1))
    y = O.conv_dft(np.ones((1, 1, n0, n1)), u[None, None], np.ones((1, 1, n0, n1)), S, (n0, n1))[0, 0]
    rows = np.stack([np.convolve(u[i], K1)[n1 - 1: 2 * n1 - 1] for i in range(n0)])
    want = np.stack([np.convolve(rows[:, j], K0)[n0 - 1: 2 * n0 - 1] for j in range(n1)], axis=1)
    assert np.max(np.abs(y - want)) < 1e-12 * np.max(np.abs(want))


@pytest.mark.parametrize("P", [2, 8, 16, 64, 512])
def test_dft_matrix_matches_numpy_fft(P):
    rng = np.random.default_rng(P)
    x = rng.standard_normal(P) + 1j * rng.standard_normal(P)
    assert np.max(np.abs(O.dft_matrix(P) @ x - np.fft.fft(x))) < 1e-10 * np.sqrt(P)


def test_spectrum_matches_numpy_rfftn():
    dims = (4, 6, 5)
    rng = np.random.default_rng(2)
    K = rng.standard_normal((2,) + tuple(2 * n - 1 for n in dims))
    Kp = O.wrap_place(K, dims)
    want = np.fft.rfftn(Kp, axes=(1, 2, 3)) / np.prod([2 * n for n in dims])
    got = O.spectrum_half(K, dims)
    assert np.max(np.abs(got - want)) < 1e-14


# ----------------------------------------------------------------- closed forms
@pytest.mark.parametrize("dims", [(7,), (5, 6), (3, 4, 4)])
def test_delta_kernel_gives_pointwise_product(dims):
    q, k, v, _ = _rand_problem(dims, seed=7)
    C = q.shape[1]
    K = np.zeros((C,) + tuple(2 * n - 1 for n in dims))
    K[(slice(None),) + tuple(n - 1 for n in dims)] = 1.0          # K = delta_0
    y = O.conv_dft(q, k, v, O.spectrum_full(K, dims), dims)
    assert np.max(np.abs(y - q * k * v)) < 1e-13
    assert np.array_equal(O.conv_direct(q, k, v, K, dims), q * (k * v))


@pytest.mark.parametrize("dims", [(6,), (4, 5), (3, 3, 4)])
def test_constant_kernel_gives_total_sum(dims):
    q, k, v, _ = _rand_problem(dims, seed=8)
    C = q.shape[1]
    K = np.ones((C,) + tuple(2 * n - 1 for n in dims))
    y = O.conv_dft(q, k, v, O.spectrum_full(K, dims), dims)
    axes = tuple(range(2, 2 + len(dims)))
    want = q * np.sum(k * v, axis=axes, keepdims=True)
    assert np.max(np.abs(y - want)) < 1e-12 * np.max(np.abs(want))


@pytest.mark.parametrize("dims", [(6,), (5, 4), (4, 3, 5)])
def test_shifted_delta_kernel_shifts_the_signal(dims):
    """K = delta at offset s: y[i] = q[i] u[i - s] (0 where i - s leaves the grid).
    A transposed operand or a correlation instead of a convolution fails this."""
    q, k, v, _ = _rand_problem(dims, seed=9)
    C = q.shape[1]
    s = tuple(1 if a % 2 == 0 else -2 for a in range(len(dims)))
    K = np.zeros((C,) + tuple(2 * n - 1 for n in dims))
    K[(slice(None),) + tuple(n - 1 + sa for n, sa in zip(dims, s))] = 1.0
    y = O.conv_dft(q, k, v, O.spectrum_full(K, dims), dims)
    u = k * v
    want = np.zeros_like(u)
    src = tuple(slice(max(0, -sa), n - max(0, sa)) for n, sa in zip(dims, s))
    dst = tuple(slice(max(0, sa), n - max(0, -sa)) for n, sa in zip(dims, s))
    want[(slice(None), slice(None)) + dst] = u[(slice(None), slice(None)) + src]
    assert np.max(np.abs(y - q * want)) < 1e-13


def test_spectrum_of_shifted_delta_is_a_phase_ramp():
    dims = (4, 6)
    t0 = (-3, 2)
    K = np.zeros((1, 7, 11))
    K[0, t0[0] + 3, t0[1] + 5] = 1.0
    S = O.spectrum_full(K, dims)[0]
    P = (8, 12)
    k0, k1 = np.meshgrid(np.arange(8), np.arange(12), indexing="ij")
    want = np.exp(-2j * np.pi * (k0 * t0[0] / P[0] + k1 * t0[1] / P[1])) / 96.0
    assert np.max(np.abs(S - want)) < 1e-15


def test_spectrum_at_points_matches_numpy_fftn():
    """The sampled definition against numpy's FFT of the wrap-placed kernel."""
    dims = (5, 4, 3)
    rng = np.random.default_rng(21)
    K = rng.standard_normal((2,) + tuple(2 * n - 1 for n in dims))
    full = np.fft.fftn(O.wrap_place(K, dims), axes=(1, 2, 3)) / np.prod([2 * n for n in dims])
    pts = np.stack([rng.integers(0, 2, 20)] + [rng.integers(0, 2 * n, 20) for n in dims], axis=1)
    got = O.spectrum_at(K, dims, pts)
    want = np.array([full[tuple(p)] for p in pts])
    assert np.max(np.abs(got - want)) < 1e-14


def test_spectrum_at_of_shifted_delta_on_a_long_axis():
    """Closed form on a 1D grid of the long-context size class: K = delta at
    t0 gives exp(-2 pi i k t0 / P) / P at every frequency k."""
    n, t0 = 4096, -1234
    K = np.zeros((1, 2 * n - 1))
    K[0, t0 + n - 1] = 1.0
    ks = np.array([0, 1, 7, n - 1, n, n + 1, 2 * n - 1])
    got = O.spectrum_at(K, (n,), np.stack([np.zeros_like(ks), ks], axis=1))
    want = np.exp(-2j * np.pi * ks * t0 / (2 * n)) / (2 * n)
    assert np.max(np.abs(got - want)) < 1e-15


def test_long_1d_direct_at_points_matches_numpy_convolve():
    """Sampled outputs of the definition on a long 1D grid against numpy's
    full linear convolution (the crop keeps indices 0..n-1 of u * K shifted by
    the kernel's centre n - 1)."""
    n = 8192
    rng = np.random.default_rng(22)
    q, k, v = (rng.standard_normal((1, 1, n)) for _ in range(3))
    K = rng.standard_normal((1, 2 * n - 1))
    full = np.convolve((k * v)[0, 0], K[0])                 # index i + n - 1 holds output i
    pts = np.array([[0, 0, i] for i in (0, 1, 777, n // 2, n - 2, n - 1)])
    got = O.conv_direct_at(q, k, v, K, (n,), pts)
    want = np.array([q[0, 0, i] * full[i + n - 1] for i in pts[:, 2]])
    assert np.max(np.abs(got - want)) < 1e-10 * np.max(np.abs(want))


# ------------------------------------------------------------------- invariants
def test_linearity_in_v():
    dims = (6, 7)
    q, k, v1, K = _rand_problem(dims, seed=12)
    _, _, v2, _ = _rand_problem(dims, seed=13)
    S = O.spectrum_full(K, dims)
    y = lambda v: O.conv_dft(q, k, v, S, dims)
    assert np.max(np.abs(y(v1 + 2 * v2) - (y(v1) + 2 * y(v2)))) < 1e-12


def test_translation_equivariance():
    """u supported in an interior box, shifted by s inside the grid:
    the unit-gated output shifts by s wherever both indices are on the grid."""
    dims = (12, 10)
    rng = np.random.default_rng(14)
    K = rng.standard_normal((1, 23, 19))
    S = O.spectrum_full(K, dims)
    u = np.zeros((1, 1) + dims)
    u[0, 0, 3:6, 2:5] = rng.standard_normal((3, 3))
    s = (4, 3)
    us = np.roll(u, s, axis=(2, 3))
    one = np.ones((1, 1) + dims)
    y = O.conv_dft(one, u, one, S, dims)[0, 0]
    ys = O.conv_dft(one, us, one, S, dims)[0, 0]
    assert np.max(np.abs(ys[s[0]:, s[1]:] - y[: dims[0] - s[0], : dims[1] - s[1]])) < 1e-12


@pytest.mark.parametrize("dims", [(8,), (6, 5)])
def test_zero_padding_gives_linear_not_circular(dims):
    """Impulse at j = 0 and K non-zero only at offset -1 (last axis): a linear
    convolution puts the response at i = -1, outside the crop, so y = 0; the
    circular convolution on the unpadded grid wraps it to i = n - 1."""
    d = len(dims)
    u = np.zeros((1, 1) + dims)
    u[(0, 0) + (0,) * d] = 1.0
    K = np.zeros((1,) + tuple(2 * n - 1 for n in dims))
    centre = [n - 1 for n in dims]
    centre[-1] -= 1
    K[(0,) + tuple(centre)] = 2.5
    one = np.ones_like(u)
    y = O.conv_dft(one, u, one, O.spectrum_full(K, dims), dims)
    assert np.max(np.abs(y)) < 1e-14
    Kper = np.zeros((1,) + dims)
    Kper[(0,) + (0,) * (d - 1) + (dims[-1] - 1,)] = 2.5
    yc = O.conv_circular(one, u, one, Kper, dims)
    want = np.zeros_like(u)
    want[(0, 0) + (0,) * (d - 1) + (dims[-1] - 1,)] = 2.5
    assert np.max(np.abs(yc - want)) < 1e-13


# ------------------------------------------------------------------ spectrum
def test_half_spectrum_hermitian_and_dc():
    dims = (6, 4)
    rng = np.random.default_rng(15)
    K = rng.standard_normal((2, 11, 7))
    Sh = O.spectrum_half(K, dims)
    S = O.spectrum_full(K, dims)
    assert np.max(np.abs(Sh[:, 0, 0] - K.sum(axis=(1, 2)) / 96.0)) < 1e-14
    P0 = 12
    for kx in (0, dims[-1]):                 # self-conjugate columns
        col = Sh[:, :, kx]
        assert np.max(np.abs(col - np.conj(col[:, np.mod(-np.arange(P0), P0)]))) < 1e-14
    assert np.max(np.abs(O.full_from_half(Sh, dims) - S)) < 1e-14


def test_wrap_place_slot_n_is_zero():
    dims = (4, 5)
    K = np.ones((1, 7, 9))
    Kp = O.wrap_place(K, dims)
    assert np.all(Kp[0, 4, :] == 0) and np.all(Kp[0, :, 5] == 0)
    assert Kp.sum() == 63 and Kp[0, 7, 9] == 1.0 and Kp[0, 3, 4] == 1.0


# ------------------------------------------------------------------- filter MLP
def _params(C, fin, H=64):
    return W.FilterParams(np.zeros((H, fin), np.float32), np.zeros(H, np.float32),
                          np.zeros((C, H), np.float32), np.zeros(C, np.float32),
                          np.zeros(C, np.float32), 8.0)


def test_filter_window_closed_form():
    dims = (8, 8)
    p = _params(2, 32)
    p.b2[:] = [1.0, -2.0]
    p.alpha[:] = [0.5, 2.0]
    K = O.implicit_kernel(p, dims)
    # offset (3, 4): ||t|| = 5; offset (0, 0): window 1
    assert abs(K[0, 7 + 3, 7 + 4] - np.exp(-0.5 * 5 / 8.0)) < 1e-15
    assert abs(K[1, 7 - 3, 7 + 4] - (-2.0) * np.exp(-2.0 * 5 / 8.0)) < 1e-15
    assert K[1, 7, 7] == -2.0


def test_filter_gaussian_window_closed_form():
    """window 1: exp(-alpha (||t|| / s)^2) (reading of the learnable Gaussian
    window); W2 = 0 isolates the window times b2."""
    dims = (8, 8, 8)
    p = _params(2, 48)
    p.W2[:] = 0.0
    p.b2[:] = [1.0, 3.0]
    p.alpha[:] = [0.5, 2.0]
    K = O.implicit_kernel(p, dims, window=1)
    # offset (1, 2, 2): ||t|| = 3, s = 8
    assert abs(K[0, 7 + 1, 7 - 2, 7 + 2] - np.exp(-0.5 * (3 / 8.0) ** 2)) < 1e-15
    assert abs(K[1, 7 - 1, 7 + 2, 7 - 2] - 3.0 * np.exp(-2.0 * (3 / 8.0) ** 2)) < 1e-15
    assert K[1, 7, 7, 7] == 3.0
    # the exponential window at the same offset differs (the two readings are distinct)
    Ke = O.implicit_kernel(p, dims, window=0)
    assert abs(Ke[0, 8, 5, 9] - np.exp(-0.5 * 3 / 8.0)) < 1e-15


@pytest.mark.parametrize("axis,m,cos", [(0, 1, 0), (1, 1, 0), (1, 3, 1), (0, 8, 1), (2, 5, 0)])
def test_filter_feature_order_closed_form(axis, m, cos):
    """One hidden unit reading one feature: K_0(t) = sin(f(pi m t_axis / n_axis))
    with f = sin or cos, so a wrong feature order, axis or frequency fails."""
    dims = (4, 8, 16)
    p = _params(1, 48)
    col = axis * 16 + (m - 1) * 2 + cos
    p.W1[5, col] = 1.0
    p.W2[0, 5] = 1.0
    K = O.implicit_kernel(p, dims)
    t = np.arange(-(dims[axis] - 1), dims[axis])
    f = np.cos if cos else np.sin
    want = np.sin(f(np.pi * m * t / dims[axis]))
    idx = [dims[a] - 1 for a in range(3)]
    sl = list(idx)
    sl[axis] = slice(None)
    assert np.max(np.abs(K[(0,) + tuple(sl)] - want)) < 1e-15


def test_filter_bias_and_second_layer():
    dims = (4, 4)
    p = _params(3, 32)
    p.b1[:] = np.float32(0.25)
    p.W2[2, :] = np.float32(0.5)
    p.b2[2] = np.float32(0.125)
    K = O.implicit_kernel(p, dims)
    want = 64 * 0.5 * np.sin(0.25) + 0.125
    assert np.max(np.abs(K[2] - want)) < 1e-13
    assert np.max(np.abs(K[0])) == 0.0


def test_film_identity_and_constant_hidden_layer():
    """FiLM pins: gamma = 1, beta = 0 is the plain network; gamma = 0 makes
    every hidden unit the constant sin(beta_h), so K_c = (W2 sin(beta) + b2)_c
    times the window (a closed form, independent of the offset features)."""
    dims = (4, 6)
    p = _params(3, 32)
    H = p.W1.shape[0]
    one, zero = np.ones(H, np.float32), np.zeros(H, np.float32)
    assert np.array_equal(O.implicit_kernel(p, dims, film=(one, zero)), O.implicit_kernel(p, dims))
    beta = np.linspace(-1.0, 1.0, H).astype(np.float32)
    K = O.implicit_kernel(p, dims, film=(zero, beta))
    t = O.offsets_grid(dims)
    r = np.sqrt(np.sum(t * t, axis=-1)) / p.decay_scale
    mlp = p.W2.astype(np.float64) @ np.sin(beta.astype(np.float64)) + p.b2
    want = mlp[:, None] * np.exp(-np.outer(p.alpha.astype(np.float64), r))
    assert np.max(np.abs(K.reshape(3, -1) - want)) < 1e-12


def test_film_by_explicit_loops():
    """One channel, a few offsets: the modulated sine layer written out unit by
    unit."""
    dims = (5,)
    rng = np.random.default_rng(31)
    H, F = 8, 16
    p = W.FilterParams(rng.standard_normal((H, F)).astype(np.float32), rng.standard_normal(H).astype(np.float32),
                       rng.standard_normal((2, H)).astype(np.float32), rng.standard_normal(2).astype(np.float32),
                       np.array([0.5, 1.5], np.float32), 4.0)
    g, b = rng.standard_normal(H).astype(np.float32), rng.standard_normal(H).astype(np.float32)
    K = O.implicit_kernel(p, dims, film=(g, b))
    for t in (-4, -1, 0, 3):
        feats = []
        for m in range(1, p.num_freqs + 1):
            feats += [np.sin(np.pi * m * t / 5), np.cos(np.pi * m * t / 5)]
        out = float(p.b2[1])
        for hh in range(H):
            pre = sum(float(p.W1[hh, f]) * feats[f] for f in range(F)) + float(p.b1[hh])
            out += float(p.W2[1, hh]) * np.sin(float(g[hh]) * pre + float(b[hh]))
        out *= np.exp(-float(p.alpha[1]) * abs(t) / p.decay_scale)
        assert abs(K[1, t + 4] - out) < 1e-12


# ----------------------------------------------------------- input generators
def test_bf16_rounding_is_round_to_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1.0 + 2 ** -9], dtype=np.float32)
    bits = W.round_to_bf16_bits(x)
    # 1+2^-8 is the midpoint between 1 and 1+2^-7: ties to even (1.0);
    # 1+3*2^-8 ties up to 1+2^-6 (even mantissa)
    assert list(bits) == [0x3F80, 0x3F80, 0x3F82, 0xC020, 0x3F80]
    assert np.array_equal(W.bf16_bits_to_f32(bits)[:1], np.array([1.0], np.float32))


def test_generators_are_deterministic_and_shaped():
    a = W.make_inputs(W.workload(0))
    b = W.make_inputs(W.workload(0))
    assert a.q.shape == (1, 4, 32, 32) and a.q.dtype == np.float32
    assert np.array_equal(a.k, b.k) and np.array_equal(a.filt.W2, b.filt.W2)
    assert a.filt.W1.shape == (64, 32) and a.filt.W2.shape == (4, 64)
    assert abs(a.filt.alpha[0] - 0.5) < 1e-7 and abs(a.filt.alpha[-1] - 5.0) < 1e-6


def test_workload_zero_full_direct_vs_dft():
    """The smallest benchmark grid end to end: O(L^2) definition against the
    padded-DFT route, on the seeded inputs."""
    inp = W.make_inputs(W.workload(0))
    dims = inp.wl.dims
    K = O.implicit_kernel(inp.filt, dims)
    q, k, v = inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v")
    y1 = O.conv_direct(q, k, v, K, dims)
    y2 = O.conv_dft(q, k, v, O.spectrum_full(K, dims), dims)
    assert O.rel_l2(y2, y1) < 1e-12


def test_rel_l2_compares_complex_values_as_complex():
    a = np.array([1.0 + 1.0j, 2.0])
    b = np.array([1.0 + 0.0j, 2.0])
    assert abs(O.rel_l2(a, b) - 1.0 / np.sqrt(5.0)) < 1e-15


# ------------------------------------------------------------------ backward
# dq = dy w, du[j] = sum_i q[i] dy[i] K[i - j], dk = v du, dv = k du (the
# gradients of L = sum dy y; blog sections on gradient flow and the autograd
# pattern).  Pinned by brute force, by the adjoint identity against the
# forward oracle, by exact finite differences of L, and by numpy's 1D convolve.
@pytest.mark.parametrize("dims", [(8,), (5,), (6, 5), (4, 7), (3, 4, 5)])
def test_adjoint_dft_equals_direct_sum(dims):
    q, k, v, K = _rand_problem(dims, seed=11)
    z = q * v
    S = O.spectrum_full(K, dims)
    assert O.rel_l2(O.corr_dft(z, S, dims), O.corr_direct(z, K, dims)) < 1e-12


def test_adjoint_direct_by_explicit_loops():
    dims = (3, 4)
    rng = np.random.default_rng(5)
    z = rng.standard_normal((1, 2) + dims)
    K = rng.standard_normal((2, 5, 7))
    du = O.corr_direct(z, K, dims)
    for c in range(2):
        for j0 in range(3):
            for j1 in range(4):
                s = sum(z[0, c, i0, i1] * K[c, i0 - j0 + 2, i1 - j1 + 3] for i0 in range(3) for i1 in range(4))
                assert abs(du[0, c, j0, j1] - s) < 1e-12


@pytest.mark.parametrize("dims", [(7,), (5, 6), (3, 4, 4)])
def test_adjoint_identity_against_the_forward(dims):
    """<conv(u), z> = <u, adj(z)> for the forward oracle's conv_direct."""
    rng = np.random.default_rng(7)
    shape = (2, 3) + dims
    u, z = rng.standard_normal(shape), rng.standard_normal(shape)
    K = rng.standard_normal((3,) + tuple(2 * n - 1 for n in dims))
    lhs = np.sum(O.conv_direct(np.ones(shape), u, np.ones(shape), K, dims) * z)
    rhs = np.sum(u * O.corr_direct(z, K, dims))
    assert abs(lhs - rhs) <= 1e-11 * max(1.0, abs(lhs))


@pytest.mark.parametrize("dims", [(8,), (6, 5), (3, 4, 5)])
def test_backward_matches_finite_differences(dims):
    """L = sum dy * y is linear in each of q, k, v, so the central difference
    along any direction is exact up to rounding."""
    q, k, v, K = _rand_problem(dims, seed=21)
    rng = np.random.default_rng(22)
    dy = rng.standard_normal(q.shape)
    S = O.spectrum_full(K, dims)
    dq, dk, dv = O.backward_dft(q, k, v, dy, S, dims)

    def L(q_, k_, v_):
        return float(np.sum(dy * O.conv_direct(q_, k_, v_, K, dims)))

    for name, g in (("q", dq), ("k", dk), ("v", dv)):
        dirn = rng.standard_normal(q.shape)
        eps = 0.5
        args_p = {"q_": q, "k_": k, "v_": v}
        args_m = dict(args_p)
        args_p[name + "_"] = args_p[name + "_"] + eps * dirn
        args_m[name + "_"] = args_m[name + "_"] - eps * dirn
        fd = (L(**args_p) - L(**args_m)) / (2 * eps)
        an = float(np.sum(g * dirn))
        assert abs(fd - an) <= 1e-10 * max(1.0, abs(an)), name


@pytest.mark.parametrize("n", [5, 8, 13])
def test_1d_adjoint_matches_numpy_convolve(n):
    """d = 1: du[j] = sum_i z[i] K[i - j] = convolve(reverse(z), K)[2(n-1) - j]."""
    rng = np.random.default_rng(n)
    z = rng.standard_normal(n)
    Kf = rng.standard_normal(2 * n - 1)
    du = O.corr_direct(z[None, None], Kf[None], (n,))[0, 0]
    want = np.convolve(z[::-1], Kf)[n - 1: 2 * n - 1][::-1]
    assert np.max(np.abs(du - want)) < 1e-12


def test_backward_direct_at_points_matches_full():
    dims = (5, 6)
    q, k, v, K = _rand_problem(dims, seed=31)
    z = q * v
    full = O.corr_direct(z, K, dims)
    pts = np.array([[1, 2, 0, 0], [0, 1, 4, 5], [1, 0, 2, 3]])
    got = O.corr_direct_at(z, K, dims, pts)
    want = np.array([full[tuple(p)] for p in pts])
    assert np.max(np.abs(got - want)) < 1e-12


@pytest.mark.parametrize("dims", [(7,), (4, 6), (3, 3, 4)])
def test_backward_direct_equals_dft_route(dims):
    """The two backward routes (direct sums on the grid, and padded DFTs with
    the conjugate spectrum) agree: a sign or index slip in the adjoint of
    either fails here."""
    q, k, v, K = _rand_problem(dims, seed=61)
    dy = np.random.default_rng(62).standard_normal(q.shape)
    a = O.backward_direct(q, k, v, dy, K, dims)
    b = O.backward_dft(q, k, v, dy, O.spectrum_full(K, dims), dims)
    for x, y in zip(a, b):
        assert np.max(np.abs(x - y)) < 1e-11 * max(1.0, np.max(np.abs(y)))


def test_reference_output_is_the_definition_on_the_smallest_workload():
    """The convenience route used by the GPU tests (implicit kernel -> spectrum
    -> DFT convolution) equals the direct sum with the same kernel."""
    wl = W.custom((6, 5), 1, 2, seed=63)
    inp = W.make_inputs(wl)
    K = O.implicit_kernel(inp.filt, wl.dims)
    want = O.conv_direct(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), K, wl.dims)
    assert np.max(np.abs(O.reference_output(inp) - want)) < 1e-11 * np.max(np.abs(want))


# ------------------------------------------------------ kernel-value gradient
@pytest.mark.parametrize("dims", [(6,), (4, 5), (3, 4, 3)])
def test_kernel_grad_dft_equals_direct(dims):
    q, k, v, _ = _rand_problem(dims, seed=51)
    dy = np.random.default_rng(52).standard_normal(q.shape)
    a = O.kernel_grad_dft(q, k, v, dy, dims)
    b = O.kernel_grad_direct(q, k, v, dy, dims)
    assert O.rel_l2(a, b) < 1e-12


@pytest.mark.parametrize("dims", [(7,), (5, 4), (3, 3, 4)])
def test_kernel_grad_matches_finite_differences(dims):
    """L = sum dy y is linear in K: the central difference along a random
    direction of K is exact up to rounding."""
    q, k, v, K = _rand_problem(dims, seed=61)
    rng = np.random.default_rng(62)
    dy = rng.standard_normal(q.shape)
    g = O.kernel_grad_direct(q, k, v, dy, dims)
    D = rng.standard_normal(K.shape)

    def L(KK):
        return float(np.sum(dy * O.conv_direct(q, k, v, KK, dims)))

    fd = (L(K + 0.5 * D) - L(K - 0.5 * D)) / 1.0
    an = float(np.sum(g * D))
    assert abs(fd - an) <= 1e-10 * max(1.0, abs(an))


def test_kernel_grad_by_explicit_loops():
    dims = (3, 4)
    q, k, v, _ = _rand_problem(dims, B=2, C=1, seed=71)
    dy = np.random.default_rng(72).standard_normal(q.shape)
    g = O.kernel_grad_direct(q, k, v, dy, dims)
    for t0 in range(-2, 3):
        for t1 in range(-3, 4):
            s = 0.0
            for b in range(2):
                for i0 in range(3):
                    for i1 in range(4):
                        j0, j1 = i0 - t0, i1 - t1
                        if 0 <= j0 < 3 and 0 <= j1 < 4:
                            s += q[b, 0, i0, i1] * dy[b, 0, i0, i1] * k[b, 0, j0, j1] * v[b, 0, j0, j1]
            assert abs(g[0, t0 + 2, t1 + 3] - s) < 1e-12


def test_kernel_grad_at_points_matches_full():
    dims = (5, 6)
    q, k, v, _ = _rand_problem(dims, seed=81)
    dy = np.random.default_rng(82).standard_normal(q.shape)
    full = O.kernel_grad_direct(q, k, v, dy, dims)
    pts = np.array([[0, -4, 5], [2, 0, 0], [1, 3, -2]])
    got = O.kernel_grad_at(q, k, v, dy, dims, pts)
    want = np.array([full[p[0], p[1] + 4, p[2] + 5] for p in pts])
    assert np.max(np.abs(got - want)) < 1e-12


# -------------------------------------------------------------- circular mode
@pytest.mark.parametrize("dims", [(8,), (4, 6), (4, 2, 4)])
def test_circular_equals_linear_with_periodized_kernel(dims):
    """sum_j u[j] Kper[(i - j) mod n] = sum_j u[j] K_lin[i - j] for i, j in
    [0, n): the circular DFT route against the linear direct sum."""
    rng = np.random.default_rng(91)
    shape = (2, 3) + dims
    q, k, v = (rng.standard_normal(shape) for _ in range(3))
    Kper = rng.standard_normal((3,) + dims)
    yc = O.conv_circular(q, k, v, Kper, dims)
    yl = O.conv_direct(q, k, v, O.periodize_to_offsets(Kper, dims), dims)
    assert O.rel_l2(yc, yl) < 1e-12


def test_circular_direct_by_explicit_loops():
    dims = (3, 4)
    rng = np.random.default_rng(92)
    q, k, v = (rng.standard_normal((1, 1) + dims) for _ in range(3))
    Kper = rng.standard_normal((1,) + dims)
    y = O.conv_circular(q, k, v, Kper, dims)
    for i0 in range(3):
        for i1 in range(4):
            s = sum(k[0, 0, j0, j1] * v[0, 0, j0, j1] * Kper[0, (i0 - j0) % 3, (i1 - j1) % 4]
                    for j0 in range(3) for j1 in range(4))
            assert abs(y[0, 0, i0, i1] - q[0, 0, i0, i1] * s) < 1e-12


def test_periodic_kernel_takes_the_centred_representative():
    dims = (8, 4)
    p = _params(2, 32)
    Kp = O.implicit_kernel_periodic(p, dims)
    K = O.implicit_kernel(p, dims)
    # tau = (5, 3) -> representatives (-3, -1)
    assert np.array_equal(Kp[:, 5, 3], K[:, 7 - 3, 3 - 1])
    # tau = (4, 2) -> (-4, -2): the half-way offset is taken as negative
    assert np.array_equal(Kp[:, 4, 2], K[:, 7 - 4, 3 - 2])
    assert np.array_equal(Kp[:, 0, 0], K[:, 7, 3])


@pytest.mark.parametrize("dims", [(6,), (4, 3)])
def test_periodic_kernel_grad_folds_the_linear_one(dims):
    """dKper[tau] = sum over linear offsets t = tau mod n of dK[t], and it
    matches exact finite differences of the circular forward."""
    rng = np.random.default_rng(93)
    shape = (2, 2) + dims
    q, k, v, dy = (rng.standard_normal(shape) for _ in range(4))
    g = O.kernel_grad_periodic_direct(q, k, v, dy, dims)
    lin = O.kernel_grad_direct(q, k, v, dy, dims)
    fold = np.zeros_like(g)
    for t in itertools.product(*[range(-(n - 1), n) for n in dims]):
        fold[(slice(None),) + tuple(ta % n for ta, n in zip(t, dims))] += \
            lin[(slice(None),) + tuple(ta + n - 1 for ta, n in zip(t, dims))]
    assert np.max(np.abs(fold - g)) < 1e-11
    Kper = rng.standard_normal((2,) + dims)
    D = rng.standard_normal(Kper.shape)

    def L(KK):
        return float(np.sum(dy * O.conv_circular(q, k, v, KK, dims)))

    fd = (L(Kper + 0.5 * D) - L(Kper - 0.5 * D)) / 1.0
    assert abs(fd - float(np.sum(g * D))) <= 1e-10 * max(1.0, abs(fd))
