"""GPU parity: the CUDA path through the C ABI against the float64 oracle on the
same seeded inputs (relative L2 error <= 1e-4 for fp32 activations, <= 1e-2 for
bf16 activations with fp32 compute), plus invariants that hold at any size.
The operation: HyenaND blog, section "HyenaND" (output equation), and the
arXiv 2607.19378 summary, "Methodologie" (zero padding to twice the grid)."""
import numpy as np
import pytest

from dimensional_long_convolution_b200 import hyena_nd as H
from dimensional_long_convolution_b200 import workloads as W
from oracle import hyena_nd_oracle as O

from gpu_util import TOL, make_op, run, sample_points, set_filter, to_dev, to_host, torch

pytestmark = pytest.mark.gpu


def _spectrum_oracle(inp, channels=None):
    K = O.implicit_kernel(inp.filt, inp.wl.dims, channels=channels)
    return K, O.spectrum_half(K, inp.wl.dims)


# ------------------------------------------------------------- filter (call 1)
@pytest.mark.parametrize("dims,C", [((8,), 3), ((32,), 5), ((32, 32), 4), ((16, 64), 3), ((64, 64), 6),
                                    ((256, 256), 2), ((8, 16, 32), 3), ((64, 64, 64), 2), ((128, 128, 16), 2)])
def test_filter_spectrum_matches_oracle(dims, C):
    wl = W.custom(dims, 1, C, seed=11)
    inp = W.make_inputs(wl, with_qkv=False)
    op = make_op(wl)
    set_filter(op, inp.filt)
    got = to_host(op.export_spectrum())
    _, want = _spectrum_oracle(inp)
    assert got.shape == want.shape
    assert O.rel_l2(got, want) < 2e-5


@pytest.mark.parametrize("dims,C", [((32,), 3), ((16, 64), 3), ((256, 256), 2), ((16, 8, 32), 2)])
def test_filter_spectrum_gaussian_window(dims, C):
    wl = W.custom(dims, 1, C, seed=17)
    inp = W.make_inputs(wl, with_qkv=False)
    op = make_op(wl)
    t = torch()
    f = inp.filt
    op.set_filter(t.from_numpy(f.W1), t.from_numpy(f.b1), t.from_numpy(f.W2), t.from_numpy(f.b2),
                  t.from_numpy(f.alpha), f.decay_scale, f.num_freqs, window=1)
    got = to_host(op.export_spectrum())
    want = O.spectrum_half(O.implicit_kernel(f, dims, window=1), dims)
    assert O.rel_l2(got, want) < 2e-5


@pytest.mark.parametrize("i,channels", [(1, [0, 255]), (2, [0, 127]), (3, [0, 63]), (4, [0, 31])])
def test_filter_spectrum_benchmark_grids(i, channels):
    wl = W.workload(i)
    inp = W.make_inputs(wl, with_qkv=False)
    op = make_op(wl)
    set_filter(op, inp.filt)
    got = to_host(op.export_spectrum())[channels]
    if wl.ndim == 3:
        # dense-DFT oracle spectrum is heavy at 256^3: check one channel
        channels = channels[:1]
        got = got[:1]
    _, want = _spectrum_oracle(inp, channels)
    assert O.rel_l2(got, want) < 2e-5


@pytest.mark.parametrize("dims,C", [((16,), 3), ((8, 8), 2), ((32, 16), 3), ((256, 8), 1), ((8, 8, 8), 2),
                                    ((16, 8, 32), 2)])
def test_spectrum_import_export_roundtrip(dims, C):
    rng = np.random.default_rng(3)
    wl = W.custom(dims, 1, C)
    op = make_op(wl)
    shape = op.natural_shape()
    nat = (rng.standard_normal(shape) + 1j * rng.standard_normal(shape)).astype(np.complex64)
    op.import_spectrum(torch().from_numpy(nat))
    back = to_host(op.export_spectrum())
    assert np.max(np.abs(back - nat)) < 1e-6 * np.max(np.abs(nat))


# ------------------------------------------------------ convolution (call 2/3)
SMALL = [
    ((8,), 3, 5, "f32"), ((32,), 2, 3, "f32"), ((64,), 1, 7, "bf16"), ((256,), 3, 3, "f32"),
    ((8, 8), 2, 3, "f32"), ((16, 32), 2, 2, "f32"), ((32, 16), 1, 3, "bf16"), ((64, 64), 2, 3, "f32"),
    ((8, 128), 1, 2, "f32"), ((128, 128), 1, 2, "f32"), ((128, 8), 2, 1, "bf16"),
    ((256, 64), 1, 2, "f32"), ((64, 256), 2, 1, "bf16"), ((256, 256), 1, 1, "f32"),
    ((8, 8, 8), 2, 2, "f32"), ((16, 8, 32), 1, 3, "f32"), ((32, 32, 32), 1, 2, "bf16"),
    ((16, 16, 128), 2, 2, "f32"), ((64, 64, 8), 1, 2, "bf16"), ((8, 8, 256), 3, 2, "f32"),
    ((8, 16, 256), 1, 2, "f32"), ((128, 128, 16), 1, 2, "f32"), ((64, 128, 8), 2, 1, "f32"),
]


@pytest.mark.parametrize("dims,B,C,dt", SMALL)
def test_conv_matches_oracle_small(dims, B, C, dt):
    wl = W.custom(dims, B, C, io_dtype=dt, seed=sum(dims) + B + C)
    inp = W.make_inputs(wl)
    K, _ = _spectrum_oracle(inp)
    want = O.conv_dft(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), O.spectrum_full(K, dims), dims)
    got, _ = run(inp)
    assert O.rel_l2(got, want) <= TOL[dt]
    # every (b, c) volume on its own, so a wrong pair mapping cannot hide
    for b in range(B):
        for c in range(C):
            assert O.rel_l2(got[b, c], want[b, c]) <= 3 * TOL[dt]


@pytest.mark.parametrize("dims,B,C,dt", [((64, 64), 2, 3, "f32"), ((256, 128), 1, 2, "f32"), ((32,), 2, 3, "f32"),
                                         ((16, 16, 16), 1, 2, "f32")])
def test_conv_with_oracle_spectrum(dims, B, C, dt):
    """The oracle's own float64 spectrum imported into the CUDA path."""
    wl = W.custom(dims, B, C, io_dtype=dt, seed=5)
    inp = W.make_inputs(wl)
    K, Sh = _spectrum_oracle(inp)
    want = O.conv_dft(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), O.spectrum_full(K, dims), dims)
    got, _ = run(inp, natural_spectrum=Sh)
    assert O.rel_l2(got, want) <= TOL[dt]


@pytest.mark.parametrize("i", [0, 1])
def test_benchmark_grid_full_output(i):
    wl = W.workload(i)
    inp = W.make_inputs(wl)
    want = O.reference_output(inp)
    got, _ = run(inp)
    assert O.rel_l2(got, want) <= TOL[wl.io_dtype]


@pytest.mark.parametrize("i", [2, 3, 4])
def test_benchmark_grid_sampled_outputs(i):
    """Full-size grids in the benchmark's launch configuration; the oracle's
    direct sum evaluated at sampled outputs (corners included)."""
    wl = W.workload(i)
    inp = W.make_inputs(wl)
    got, _ = run(inp)
    chans = [0, wl.C - 1, wl.C // 2]
    pts = sample_points(wl, 24, seed=i, channels=chans)
    K = O.implicit_kernel(inp.filt, wl.dims, channels=chans)
    Kfull = np.zeros((wl.C,) + K.shape[1:])
    for j, c in enumerate(chans):
        Kfull[c] = K[j]
    want = O.conv_direct_at(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), Kfull, wl.dims, pts)
    gv = np.array([got[tuple(p)] for p in pts])
    assert O.rel_l2(gv, want) <= TOL[wl.io_dtype]
    assert np.all(np.isfinite(got))


# ------------------------------------------------------------------ invariants
@pytest.mark.parametrize("dims", [(32,), (64, 64), (256, 64), (16, 16, 16)])
def test_delta_kernel_gives_pointwise_product(dims):
    wl = W.custom(dims, 2, 2)
    inp = W.make_inputs(wl)
    op = make_op(wl)
    P = np.prod([2 * n for n in dims])
    nat = np.full(op.natural_shape(), 1.0 / P, dtype=np.complex64)       # spectrum of delta_0
    got, _ = run(inp, natural_spectrum=nat)
    want = inp.as_f64("q") * inp.as_f64("k") * inp.as_f64("v")
    assert np.max(np.abs(got - want)) < 1e-5 * np.max(np.abs(want))


@pytest.mark.parametrize("dims", [(64, 64), (32, 32, 32)])
def test_linearity_in_v(dims):
    wl = W.custom(dims, 1, 2, seed=9)
    a = W.make_inputs(wl)
    b = W.make_inputs(wl, seed=10)
    op = make_op(wl)
    set_filter(op, a.filt)
    y1, _ = run(a, op=op)
    b.q, b.k = a.q, a.k
    y2, _ = run(b, op=op)
    a2 = W.make_inputs(wl)
    a2.v = (a.v + 2 * b.v).astype(np.float32)
    y3, _ = run(a2, op=op)
    assert np.max(np.abs(y3 - (y1 + 2 * y2))) < 1e-4 * np.max(np.abs(y3))


def test_per_sample_spectrum_stride():
    """spectrum_batch_stride != 0: sample b uses its own spectrum set."""
    dims = (32, 32)
    wl = W.custom(dims, 2, 3, seed=21)
    inp = W.make_inputs(wl)
    t = torch()
    rng = np.random.default_rng(1)
    sets = []
    for b in range(2):
        Kb = rng.standard_normal((3,) + tuple(2 * n - 1 for n in dims))
        sets.append(Kb)
    op = make_op(wl)
    specs = []
    for Kb in sets:
        op.import_spectrum(t.from_numpy(O.spectrum_half(Kb, dims).astype(np.complex64)))
        specs.append(op.spectrum.clone())
    both = t.cat(specs)
    sbs = op.spec_bytes
    got, _ = run(inp, op=op, sbs=sbs, spectrum=both)
    for b in range(2):
        want = O.conv_dft(inp.as_f64("q")[b:b + 1], inp.as_f64("k")[b:b + 1], inp.as_f64("v")[b:b + 1],
                          O.spectrum_full(sets[b], dims), dims)
        assert O.rel_l2(got[b:b + 1], want) < 1e-4


def test_single_volume_entry_point():
    dims = (64, 64)
    wl = W.custom(dims, 1, 1, seed=4)
    inp = W.make_inputs(wl)
    op = make_op(wl)
    set_filter(op, inp.filt)
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    y = torch().empty_like(q)
    st = H.fftconv(op.p, q.data_ptr(), k.data_ptr(), v.data_ptr(), op.spectrum.data_ptr(), y.data_ptr(),
                   op.ws.data_ptr(), op.ws_bytes, op._stream())
    assert st == H.OK
    assert H.last_launch_count() == 1
    torch().cuda.synchronize()
    want = O.reference_output(inp)
    assert O.rel_l2(to_host(y), want) < 1e-4


def test_launch_counts_per_tier():
    # 1D and 2D <= 64: one fused launch; larger grids: waves of 3 launches
    cases = [((64,), 4, 4, 1), ((64, 64), 2, 2, 1), ((256, 256), 2, 2, 3), ((16, 16, 16), 1, 2, 3),
             ((128, 128, 16), 1, 2, 3)]
    for dims, B, C, want in cases:
        wl = W.custom(dims, B, C)
        inp = W.make_inputs(wl)
        run(inp)
        assert H.last_launch_count() == want, dims


def _check_sampled(wl, inp, got, chans, tol, npts=12):
    pts = sample_points(wl, npts, seed=2, channels=chans)
    K = O.implicit_kernel(inp.filt, wl.dims, channels=chans)
    Kfull = np.zeros((wl.C,) + K.shape[1:])
    for j, c in enumerate(chans):
        Kfull[c] = K[j]
    want = O.conv_direct_at(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), Kfull, wl.dims, pts)
    gv = np.array([got[tuple(p)] for p in pts])
    assert O.rel_l2(gv, want) <= tol


def _wave_edge_channels(wl):
    """Channels at the start and end of the first two waves and the last
    channel, from the library's plan (volumes run in channel-major order)."""
    info = H.plan_info(H.problem(wl.dims, wl.B, wl.C, H.BF16 if wl.io_dtype == "bf16" else H.F32))
    w = int(info["wave"])
    ords = [0, w - 1, w, 2 * w - 1, wl.B * wl.C - 1]
    return info, sorted({o // wl.B for o in ords})


def test_multi_wave_schedule_2d():
    """More volumes (400 of 256^2) than one wave's workspace holds: ten
    balanced waves of 40 volumes, round-robin on three streams."""
    dims = (256, 256)
    wl = W.custom(dims, 2, 200, io_dtype="bf16", seed=31)
    info, chans = _wave_edge_channels(wl)
    assert info["waves"] == 10 and info["streams"] == 3
    inp = W.make_inputs(wl)
    got, _ = run(inp)
    assert H.last_launch_count() == info["launches"] == 30
    _check_sampled(wl, inp, got, chans, 1e-2)


def test_multi_wave_schedule_3d():
    """100 volumes of 32x64x64 at 1 MiB of intermediate each run as five
    balanced waves of 20, round-robin on three streams."""
    dims = (32, 64, 64)
    wl = W.custom(dims, 1, 100, io_dtype="bf16", seed=37)
    info, chans = _wave_edge_channels(wl)
    assert info["waves"] == 5 and info["streams"] == 3
    inp = W.make_inputs(wl)
    got, _ = run(inp)
    assert H.last_launch_count() == info["launches"] == 15
    _check_sampled(wl, inp, got, chans, 1e-2)


def test_repeated_calls_on_one_workspace():
    """Back-to-back calls on one workspace give identical results and leave
    the device status clear."""
    dims = (32, 32, 64)
    wl = W.custom(dims, 2, 5, seed=13)
    inp = W.make_inputs(wl)
    op = make_op(wl)
    set_filter(op, inp.filt)
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    outs = [to_host(op(q, k, v)) for _ in range(3)]
    assert H.device_status(op.ws.data_ptr(), op._stream()) == H.OK
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])
    want = O.reference_output(inp)
    assert O.rel_l2(outs[0], want) < 1e-4


# ------------------------------------------------------------ device status
def test_bounded_wait_reports_timeout_and_recovers():
    t = torch()
    ws = t.zeros(4096, dtype=t.uint8, device="cuda")
    s = int(t.cuda.current_stream().cuda_stream)
    assert H.workspace_init(ws.data_ptr(), 4096, s) == H.OK
    assert H.debug_bounded_wait(ws.data_ptr(), 4096, 2000, s) == H.OK
    assert H.device_status(ws.data_ptr(), s) == H.ERR_DEVICE_TIMEOUT
    assert H.device_status(ws.data_ptr(), s) == H.OK         # cleared by the read
    # the context is still usable
    x = t.ones(16, device="cuda")
    assert float((x * 2).sum()) == 32.0


def test_calls_run_in_their_own_workspace_size():
    """The filter call in exactly hyena_nd_workspace_bytes_for(FILTER) bytes
    and the convolution in exactly ..._for(CONV) bytes (several waves on
    several streams), against the oracle."""
    t = torch()
    dims = (256, 256)
    wl = W.custom(dims, 2, 70, io_dtype="bf16", seed=45)
    inp = W.make_inputs(wl)
    op = make_op(wl)
    p = op.p
    s = int(t.cuda.current_stream().cuda_stream)
    wf = t.empty(H.workspace_bytes_for(p, H.CALL_FILTER), dtype=t.uint8, device="cuda")
    wc = t.empty(H.workspace_bytes_for(p, H.CALL_CONV), dtype=t.uint8, device="cuda")
    assert wc.numel() < op.ws_bytes
    for w in (wf, wc):
        assert H.workspace_init(w.data_ptr(), w.numel(), s) == H.OK
    f = inp.filt
    wts = [t.from_numpy(a).cuda() for a in (f.W1, f.b1, f.W2, f.b2, f.alpha)]
    fl = H.Filter()
    fl.num_freqs, fl.hidden = f.num_freqs, f.hidden
    fl.W1, fl.b1, fl.W2, fl.b2, fl.alpha = (x.data_ptr() for x in wts)
    fl.decay_scale, fl.window = f.decay_scale, 0
    assert H.filter_spectrum(p, fl, op.spectrum.data_ptr(), wf.data_ptr(), wf.numel(), s) == H.OK
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    y = t.empty_like(q)
    assert H.fftconv_batched(p, q.data_ptr(), k.data_ptr(), v.data_ptr(), op.spectrum.data_ptr(), 0, y.data_ptr(),
                             wc.data_ptr(), wc.numel(), s) == H.OK
    assert H.plan_info(p)["waves"] > 1
    t.cuda.synchronize()
    assert H.device_status(wc.data_ptr(), s) == H.OK
    _check_sampled(wl, inp, to_host(y), [0, 34, 35, 69], 1e-2)
