"""Element-wise GPU parity on the full benchmark grids, in the launch
configuration the benchmark times (the same planner, waves and tiers), against
the float64 oracle's padded-DFT convolution.

Every output of every (b, c) volume is compared on the 2D 256^2 (B2, C128,
bf16) and 3D 64^3 (B2, C64, fp32) grids; the 3D 128^3 grid (B1, C32, bf16) is
compared on four whole volumes at the ends of its waves.  The backward (dq, dk,
dv) and the kernel gradient are compared on whole 256^2 volumes of the
channels that start each wave, and of the last channel.  Tolerances: relative L2 <= 1e-4 (fp32 I/O) and
<= 1e-2 (bf16 I/O), over the whole tensor and over each volume on its own.

The operation: HyenaND blog, section "HyenaND" (output equation); the arXiv
2607.19378 summary, "Methodologie" (zero padding to twice the grid) and
"Implementation: nSubQ" (forward FFT, spectral modulation, inverse FFT, crop).
The oracle is evaluated channel chunk by channel chunk only to bound host
memory; every chunk runs the oracle's unchanged routines."""
import numpy as np
import pytest

from dimensional_long_convolution_b200 import hyena_nd as H
from dimensional_long_convolution_b200 import workloads as W
from oracle import hyena_nd_oracle as O

from gpu_util import TOL, make_op, run, set_filter, to_dev, to_host, torch

pytestmark = pytest.mark.gpu


def _f64(a):
    return W.bf16_bits_to_f32(a).astype(np.float64) if a.dtype == np.uint16 else a.astype(np.float64)


def _oracle_conv(inp, chans, K=None):
    """Oracle y[:, chans] (float64) for the seeded workload ``inp``; ``K``, if
    given, holds the kernels of exactly these channels."""
    dims = inp.wl.dims
    if K is None:
        K = O.implicit_kernel(inp.filt, dims, channels=list(chans))
    S = O.spectrum_full(K, dims)
    sl = (slice(None), np.asarray(chans))
    return O.conv_dft(inp.as_f64("q")[sl], inp.as_f64("k")[sl], inp.as_f64("v")[sl], S, dims)


def _check_volumes(got, want, tol, what):
    """Whole-tensor and per-volume relative L2 of got[b, c] against want."""
    assert got.shape == want.shape, what
    assert np.all(np.isfinite(got)), what
    assert O.rel_l2(got, want) <= tol, what
    worst = 0.0
    for b in range(got.shape[0]):
        for c in range(got.shape[1]):
            e = O.rel_l2(got[b, c], want[b, c])
            worst = max(worst, e)
            assert e <= tol, (what, b, c, e)
    return worst


def _plan(wl):
    return H.plan_info(H.problem(wl.dims, wl.B, wl.C, H.BF16 if wl.io_dtype == "bf16" else H.F32))


@pytest.mark.parametrize("i,chunk", [(2, 16), (3, 4)])
def test_full_grid_every_volume(i, chunk):
    """All B*C volumes of the 256^2 and 64^3 grids, element by element."""
    wl = W.workload(i)
    inp = W.make_inputs(wl)
    got, _ = run(inp)
    tol = TOL[wl.io_dtype]
    K = O.implicit_kernel(inp.filt, wl.dims)         # the hidden layer once for every channel
    for c0 in range(0, wl.C, chunk):
        chans = range(c0, min(wl.C, c0 + chunk))
        want = _oracle_conv(inp, chans, K[c0:c0 + len(chans)])
        _check_volumes(got[:, c0:c0 + len(chans)], want, tol, (wl.name, c0))


def test_full_grid_large_volume_wave_edges():
    """Whole 128^3 volumes at the edges of the waves (B = 1: the first and
    last volume of the first wave, the first of the second and the third
    waves, which run on other streams), a middle channel and the last one."""
    wl = W.workload(4)
    info = _plan(wl)
    wave = int(info["wave"])
    assert info["waves"] >= 3
    chans = sorted({0, wave - 1, wave, 2 * wave, wl.C // 2, wl.C - 1})
    inp = W.make_inputs(wl)
    got, _ = run(inp)
    for c in chans:
        want = _oracle_conv(inp, [c])
        _check_volumes(got[:, c:c + 1], want, TOL["bf16"], (wl.name, c))


def _wave_channels(wl):
    """The first channel of every wave of a convolution (waves hold whole
    channels' samples) and the last channel, from the library's plan."""
    w = int(_plan(wl)["wave"])
    firsts = {o // wl.B for o in range(0, wl.B * wl.C, w)}
    return sorted(firsts | {wl.C - 1})


def test_backward_full_volumes():
    wl = W.workload(2)
    inp = W.make_inputs(wl)
    dy = W.make_inputs(wl, seed=wl.seed + 7).q
    op = make_op(wl)
    set_filter(op, inp.filt)
    q, k, v, g = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), to_dev(dy)
    dq, dk, dv = op.backward(q, k, v, g)
    torch().cuda.synchronize()
    assert op.status() == H.OK
    chans = _wave_channels(wl)
    got = [to_host(x)[:, chans] for x in (dq, dk, dv)]
    ch = np.asarray(chans)
    K = O.implicit_kernel(inp.filt, wl.dims, channels=chans)
    S = O.spectrum_full(K, wl.dims)
    sl = (slice(None), ch)
    want = O.backward_dft(inp.as_f64("q")[sl], inp.as_f64("k")[sl], inp.as_f64("v")[sl], _f64(dy)[sl], S,
                          wl.dims)
    for name, gg, ww in zip(("dq", "dk", "dv"), got, want):
        _check_volumes(gg, ww, TOL["bf16"], name)


def test_kernel_grad_full_channels():
    """dK at every offset of the channels that start each wave and of the last
    channel (all their samples)."""
    wl = W.workload(2)
    inp = W.make_inputs(wl)
    dy = W.make_inputs(wl, seed=wl.seed + 9).q
    op = make_op(wl)
    dK = op.kernel_grad(to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), to_dev(dy))
    torch().cuda.synchronize()
    assert op.status() == H.OK
    chans = _wave_channels(wl)
    got = dK.cpu().numpy().astype(np.float64)[chans]
    sl = (slice(None), np.asarray(chans))
    want = O.kernel_grad_dft(inp.as_f64("q")[sl], inp.as_f64("k")[sl], inp.as_f64("v")[sl], _f64(dy)[sl],
                             wl.dims)
    assert got.shape == want.shape
    assert O.rel_l2(got, want) <= TOL["bf16"]
    for j in range(len(chans)):
        assert O.rel_l2(got[j], want[j]) <= TOL["bf16"], chans[j]
