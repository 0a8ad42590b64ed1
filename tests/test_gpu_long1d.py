"""GPU parity of the long 1D context tier (n from 512 to 2^26) against the
float64 oracle: the padded length-2n transform runs as a split into two or
three passes of at most 512 points, volumes go through the workspace in waves.
Forward, backward, kernel gradient, the filter spectrum and its import/export,
per-sample spectra, circular mode and the Gaussian window are each checked,
fully at sizes the dense-DFT oracle finishes quickly and on sampled outputs
(direct sums) at the longest grids.  (arXiv 2607.19378 summary: 1D sequences
are the d = 1 case of the zero-padded FFT path; blog "Native
multi-dimensional subquadratic operators via input-dependent long
convolutions", section "HyenaND".)"""
import numpy as np
import pytest

from dimensional_long_convolution_b200 import hyena_nd as H
from dimensional_long_convolution_b200 import workloads as W
from oracle import hyena_nd_oracle as O

from gpu_util import TOL, make_op, run, sample_points, set_filter, to_dev, to_host, torch

pytestmark = pytest.mark.gpu

WAVE_BYTES = 48 << 20          # the library's budget of padded complex grids in flight


def _f64(a):
    return W.bf16_bits_to_f32(a).astype(np.float64) if a.dtype == np.uint16 else a.astype(np.float64)


def _waves(n, B, C):
    """Channels 2j and 2j + 1 of a sample share one padded complex grid.
    When the grids need several waves and three fit the budget, the waves
    alternate over three streams, each in a third of the budget."""
    per = 2 * n * 8
    grids = B * ((C + 1) // 2)
    w = max(1, min(WAVE_BYTES // per, grids))
    if w < grids and 3 * per <= WAVE_BYTES:
        w = max(1, min(WAVE_BYTES // 3 // per, grids))
    return -(-grids // w)


def _per_wave(n):
    """Fused passes of one wave: 2m - 1 for a split into m = 2 or 3 levels."""
    return 3 if 2 * n <= 1 << 18 else 5


def _kernel_for(filt, dims, C, chans, window=0):
    """The oracle kernel for the sampled channels, zero elsewhere."""
    K = O.implicit_kernel(filt, dims, channels=chans, window=window)
    full = np.zeros((C,) + K.shape[1:])
    for j, c in enumerate(chans):
        full[c] = K[j]
    return full


FULL = [((512,), 2, 3, "f32"), ((512,), 1, 4, "bf16"), ((1024,), 2, 2, "f32"), ((1024,), 1, 3, "bf16")]


@pytest.mark.parametrize("dims,B,C,dt", FULL)
def test_long1d_forward_matches_oracle(dims, B, C, dt):
    wl = W.custom(dims, B, C, io_dtype=dt, seed=dims[0] + B + C)
    inp = W.make_inputs(wl)
    got, _ = run(inp)
    assert H.last_launch_count() == _per_wave(dims[0]) * _waves(dims[0], B, C)
    assert O.rel_l2(got, O.reference_output(inp)) <= TOL[dt]


@pytest.mark.parametrize("n,B,C,dt", [(65536, 2, 60, "f32"), (131072, 1, 4, "bf16"), (16384, 3, 5, "f32"),
                                     (1 << 19, 3, 7, "bf16"), (1 << 20, 1, 64, "bf16")])
def test_long1d_forward_sampled(n, B, C, dt):
    """Longest grids and multi-wave schedules, sampled outputs against direct
    sums.  2^19 tokens, B = 3, C = 7: 12 channel-pair grids of 8 MiB, so six
    waves of two on three streams, and the last pair of every sample holds
    one channel (channels 0, 3 and 6 are sampled: both halves of a pair and
    the lone channel).  2^20 tokens, B = 1, C = 64 is the benchmark's long
    1D line in its own launch configuration (32 waves of one grid on three
    streams)."""
    wl = W.custom((n,), B, C, io_dtype=dt, seed=n % 97 + C)
    inp = W.make_inputs(wl)
    got, _ = run(inp)
    assert H.last_launch_count() == _per_wave(n) * _waves(n, B, C)
    chans = sorted({0, C - 1, C // 2})
    pts = sample_points(wl, 12, seed=3, channels=chans)
    K = _kernel_for(inp.filt, wl.dims, C, chans)
    want = O.conv_direct_at(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), K, wl.dims, pts)
    gv = np.array([got[tuple(p)] for p in pts])
    assert O.rel_l2(gv, want) <= TOL[dt]


@pytest.mark.parametrize("dims,C", [((512,), 3), ((4096,), 2), ((131072,), 2)])
def test_long1d_filter_spectrum(dims, C):
    wl = W.custom(dims, 1, C, seed=13)
    inp = W.make_inputs(wl, with_qkv=False)
    op = make_op(wl)
    set_filter(op, inp.filt)
    got = to_host(op.export_spectrum())
    assert got.shape == (C, dims[0] + 1)
    K = O.implicit_kernel(inp.filt, dims)
    if dims[0] <= 1024:
        assert O.rel_l2(got, O.spectrum_half(K, dims)) < 2e-5
    rng = np.random.default_rng(5)
    ks = np.concatenate([[0, 1, dims[0] - 1, dims[0]], rng.integers(0, dims[0] + 1, 12)])
    pts = np.stack([np.arange(ks.size) % C, ks], axis=1)
    want = O.spectrum_at(K, dims, pts)
    gv = np.array([got[int(c), int(k)] for c, k in pts])
    assert O.rel_l2(gv, want) < 2e-5


def test_long1d_import_export_roundtrip_and_conv():
    """A random kernel's natural half spectrum goes in, comes back unchanged
    up to the two float32 roundings of the channel-pair layout ((K_a + K_b)/2
    and (K_a - K_b)/2 in, their sum and difference out), and drives a
    convolution equal to the oracle's with that kernel.  C = 3 leaves the
    second pair half empty."""
    dims, B, C = (1024,), 2, 3
    rng = np.random.default_rng(8)
    K = rng.standard_normal((C, 2 * dims[0] - 1)) / 64.0
    nat = O.spectrum_half(K, dims)
    wl = W.custom(dims, B, C, seed=19)
    inp = W.make_inputs(wl)
    op = make_op(wl)
    op.import_spectrum(torch().from_numpy(nat.astype(np.complex64)))
    back = to_host(op.export_spectrum())
    assert np.max(np.abs(back - nat.astype(np.complex64))) <= 4e-7 * np.max(np.abs(nat))
    got, _ = run(inp, op=op)
    want = O.conv_direct(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), K, dims)
    assert O.rel_l2(got, want) <= TOL["f32"]


def test_long1d_per_sample_spectrum():
    dims, B, C = (512,), 2, 2
    wl = W.custom(dims, B, C, seed=23)
    inp = W.make_inputs(wl)
    rng = np.random.default_rng(9)
    Ks = [rng.standard_normal((C, 2 * dims[0] - 1)) / 32.0 for _ in range(B)]
    op = make_op(wl)
    specs = []
    for Kb in Ks:
        op.import_spectrum(torch().from_numpy(O.spectrum_half(Kb, dims).astype(np.complex64)))
        specs.append(op.spectrum.clone())
    both = torch().cat(specs)
    got, _ = run(inp, op=op, spectrum=both, sbs=op.spec_bytes)
    for b in range(B):
        sl = slice(b, b + 1)
        want = O.conv_direct(inp.as_f64("q")[sl], inp.as_f64("k")[sl], inp.as_f64("v")[sl], Ks[b], dims)
        assert O.rel_l2(got[sl], want) <= TOL["f32"], b


@pytest.mark.parametrize("dims,B,C,dt", FULL[:3])
def test_long1d_backward_matches_oracle(dims, B, C, dt):
    wl = W.custom(dims, B, C, io_dtype=dt, seed=dims[0] + 31)
    inp = W.make_inputs(wl)
    dy = W.make_inputs(wl, seed=wl.seed + 7).q
    op = make_op(wl)
    set_filter(op, inp.filt)
    dq, dk, dv = op.backward(to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), to_dev(dy))
    torch().cuda.synchronize()
    assert op.status() == H.OK
    assert H.last_launch_count() == 2 * _per_wave(dims[0]) * _waves(dims[0], B, C)
    S = O.spectrum_full(O.implicit_kernel(inp.filt, dims), dims)
    want = O.backward_dft(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), _f64(dy), S, dims)
    for name, g, w in zip(("dq", "dk", "dv"), (dq, dk, dv), want):
        assert O.rel_l2(to_host(g), w) <= TOL[dt], name


def test_long1d_backward_sampled_longest():
    n, B, C = 131072, 1, 3
    wl = W.custom((n,), B, C, io_dtype="bf16", seed=37)
    inp = W.make_inputs(wl)
    dy = W.make_inputs(wl, seed=wl.seed + 7).q
    op = make_op(wl)
    set_filter(op, inp.filt)
    dq, dk, dv = (to_host(x) for x in op.backward(to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), to_dev(dy)))
    torch().cuda.synchronize()
    assert op.status() == H.OK
    chans = [0, 2]
    pts = sample_points(wl, 10, seed=6, channels=chans)
    K = _kernel_for(inp.filt, wl.dims, C, chans)
    q, k, v, g = inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), _f64(dy)
    w = O.conv_direct_at(np.ones_like(q), k, v, K, wl.dims, pts)
    du = O.corr_direct_at(q * g, K, wl.dims, pts)
    idx = [tuple(p) for p in pts]
    wants = (np.array([g[i] for i in idx]) * w, np.array([v[i] for i in idx]) * du,
             np.array([k[i] for i in idx]) * du)
    for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), wants):
        assert O.rel_l2(np.array([got[i] for i in idx]), want) <= TOL["bf16"], name


@pytest.mark.parametrize("dims,B,C,dt", [((512,), 2, 3, "f32"), ((1024,), 1, 2, "bf16")])
def test_long1d_kernel_grad_matches_oracle(dims, B, C, dt):
    wl = W.custom(dims, B, C, io_dtype=dt, seed=dims[0] + 41)
    inp = W.make_inputs(wl)
    dy = W.make_inputs(wl, seed=wl.seed + 9).q
    op = make_op(wl)
    dK = to_host(op.kernel_grad(to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), to_dev(dy)))
    torch().cuda.synchronize()
    assert op.status() == H.OK
    want = O.kernel_grad_dft(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), _f64(dy), dims)
    assert dK.shape == want.shape
    assert O.rel_l2(dK, want) <= TOL[dt]


def test_long1d_kernel_grad_sampled_several_chunks():
    """131072 points, B = 2: 6 MiB of grids a channel (two packed volumes and
    one accumulator), so 100 channels take three chunks (42, 42, 16) of the
    256 MiB kernel-gradient budget."""
    n, B, C = 131072, 2, 100
    wl = W.custom((n,), B, C, seed=43)
    inp = W.make_inputs(wl)
    dy = W.make_inputs(wl, seed=wl.seed + 9).q
    op = make_op(wl)
    dK = to_host(op.kernel_grad(to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), to_dev(dy)))
    torch().cuda.synchronize()
    assert op.status() == H.OK
    rng = np.random.default_rng(12)
    pts = np.stack([rng.integers(0, C, 14), rng.integers(-(n - 1), n, 14)], axis=1)
    pts[0] = [0, 0]
    pts[1] = [C - 1, n - 1]
    pts[2] = [42, -(n - 1)]
    pts[3] = [85, 5]
    want = O.kernel_grad_at(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), _f64(dy), wl.dims, pts)
    gv = np.array([dK[int(c), int(t) + n - 1] for c, t in pts])
    assert O.rel_l2(gv, want) <= TOL["f32"]


@pytest.mark.parametrize("dims,B,C,dt", [((1024,), 2, 2, "f32"), ((2048,), 1, 2, "bf16")])
def test_long1d_circular(dims, B, C, dt):
    wl = W.custom(dims, B, C, io_dtype=dt, seed=dims[0] + 47)
    inp = W.make_inputs(wl)
    op = H.HyenaND(dims, B, C, dt, device="cuda", circular=1)
    set_filter(op, inp.filt)
    got, _ = run(inp, op=op)
    Kper = O.implicit_kernel_periodic(inp.filt, dims)
    want = O.conv_circular(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), Kper, dims)
    assert O.rel_l2(got, want) <= TOL[dt]
    dy = W.make_inputs(wl, seed=wl.seed + 9).q
    dK = to_host(op.kernel_grad(to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), to_dev(dy)))
    torch().cuda.synchronize()
    wantK = O.kernel_grad_periodic_direct(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), _f64(dy), dims)
    assert dK.shape == wantK.shape
    assert O.rel_l2(dK, wantK) <= TOL[dt]


def test_long1d_gaussian_window_sampled():
    n, B, C = 8192, 1, 3
    wl = W.custom((n,), B, C, seed=53)
    inp = W.make_inputs(wl)
    op = make_op(wl)
    t = torch()
    f = inp.filt
    op.set_filter(t.from_numpy(f.W1), t.from_numpy(f.b1), t.from_numpy(f.W2), t.from_numpy(f.b2),
                  t.from_numpy(f.alpha), f.decay_scale, f.num_freqs, window=1)
    got, _ = run(inp, op=op)
    chans = [0, 1, 2]
    pts = sample_points(wl, 9, seed=8, channels=chans)
    K = _kernel_for(f, wl.dims, C, chans, window=1)
    want = O.conv_direct_at(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), K, wl.dims, pts)
    assert O.rel_l2(np.array([got[tuple(p)] for p in pts]), want) <= TOL["f32"]


# ------------------------------------------------ three-level split (n > 2^17)
@pytest.mark.parametrize("n,B,C,dt", [(1 << 18, 1, 2, "f32"), (1 << 19, 2, 1, "bf16")])
def test_long1d_three_levels_forward_sampled(n, B, C, dt):
    wl = W.custom((n,), B, C, io_dtype=dt, seed=61 + C)
    inp = W.make_inputs(wl)
    got, _ = run(inp)
    assert H.last_launch_count() == _per_wave(n) * _waves(n, B, C)
    chans = list(range(C))
    pts = sample_points(wl, 10, seed=9, channels=chans)
    K = _kernel_for(inp.filt, wl.dims, C, chans)
    want = O.conv_direct_at(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), K, wl.dims, pts)
    assert O.rel_l2(np.array([got[tuple(p)] for p in pts]), want) <= TOL[dt]


def test_long1d_three_levels_spectrum_backward_and_kernel_grad():
    n, B, C = 1 << 18, 2, 2
    wl = W.custom((n,), B, C, seed=67)
    inp = W.make_inputs(wl)
    dy = W.make_inputs(wl, seed=wl.seed + 7).q
    op = make_op(wl)
    set_filter(op, inp.filt)
    K = O.implicit_kernel(inp.filt, wl.dims)
    spec = to_host(op.export_spectrum())
    rng = np.random.default_rng(10)
    ks = np.concatenate([[0, 1, n - 1, n], rng.integers(0, n + 1, 8)])
    sp = np.stack([np.arange(ks.size) % C, ks], axis=1)
    assert O.rel_l2(np.array([spec[int(c), int(k)] for c, k in sp]), O.spectrum_at(K, wl.dims, sp)) < 2e-5
    q, k, v, g = (to_dev(a) for a in (inp.q, inp.k, inp.v, dy))
    dq, dk, dv = (to_host(x) for x in op.backward(q, k, v, g))
    dK = to_host(op.kernel_grad(q, k, v, g))
    torch().cuda.synchronize()
    assert op.status() == H.OK
    qf, kf, vf, gf = inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), _f64(dy)
    pts = sample_points(wl, 8, seed=11)
    w = O.conv_direct_at(np.ones_like(qf), kf, vf, K, wl.dims, pts)
    du = O.corr_direct_at(qf * gf, K, wl.dims, pts)
    idx = [tuple(p) for p in pts]
    wants = (np.array([gf[i] for i in idx]) * w, np.array([vf[i] for i in idx]) * du,
             np.array([kf[i] for i in idx]) * du)
    for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), wants):
        assert O.rel_l2(np.array([got[i] for i in idx]), want) <= TOL["f32"], name
    kp = np.stack([rng.integers(0, C, 8), rng.integers(-(n - 1), n, 8)], axis=1)
    kp[0] = [0, n - 1]
    kp[1] = [1, -(n - 1)]
    wantK = O.kernel_grad_at(qf, kf, vf, gf, wl.dims, kp)
    assert O.rel_l2(np.array([dK[int(c), int(t) + n - 1] for c, t in kp]), wantK) <= TOL["f32"]


def test_long1d_eight_million_tokens_sampled():
    """2^23 tokens (the pages' long-context class of about ten million), the
    filter network evaluated on all 2^24 - 1 offsets, sampled outputs."""
    n = 1 << 23
    wl = W.custom((n,), 1, 1, seed=71)
    inp = W.make_inputs(wl)
    got, _ = run(inp)
    pts = sample_points(wl, 6, seed=12, channels=[0])
    K = O.implicit_kernel(inp.filt, wl.dims)
    want = O.conv_direct_at(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), K, wl.dims, pts)
    assert O.rel_l2(np.array([got[tuple(p)] for p in pts]), want) <= TOL["f32"]


def test_long1d_longest_grid_shifted_delta():
    """n = 2^26, the largest grid: the natural spectrum of a delta at offset t0
    (its closed form exp(-2 pi i k t0 / P) / P) must shift the gated input,
    y[i] = q[i] u[i - t0], at every output."""
    n, t0 = 1 << 26, 12345
    wl = W.custom((n,), 1, 1, seed=73)
    inp = W.make_inputs(wl)
    op = make_op(wl)
    kk = np.arange(n + 1, dtype=np.float64)
    ph = np.mod(kk * t0, 2 * n) / (2 * n)
    nat = (np.exp(-2j * np.pi * ph) / (2 * n)).astype(np.complex64)[None]
    op.import_spectrum(torch().from_numpy(nat))
    del nat, kk, ph
    got, _ = run(inp, op=op)
    assert H.last_launch_count() == _per_wave(n)
    u = inp.as_f64("k")[0, 0] * inp.as_f64("v")[0, 0]
    want = np.zeros(n)
    want[t0:] = u[: n - t0]
    want *= inp.as_f64("q")[0, 0]
    assert O.rel_l2(got[0, 0], want) <= TOL["f32"]
