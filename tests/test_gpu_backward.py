"""GPU parity of the backward call against the float64 oracle: for a loss
gradient dy, dq = dy w, du = K (adjoint) (q dy), dk = v du, dv = k du, on every
tier (1D rows, fused 2D, multi-pass 2D and 3D incl. the 2-CTA slab pair), with
the full sampled check at the benchmark size and per-sample spectra.
(Blog "Native multi-dimensional subquadratic operators via input-dependent
long convolutions", gradient-flow and autograd sections: the backward
recomputes the FFT convolution; the adjoint uses the conjugate spectrum.)"""
import numpy as np
import pytest

from dimensional_long_convolution_b200 import hyena_nd as H
from dimensional_long_convolution_b200 import workloads as W
from oracle import hyena_nd_oracle as O

from gpu_util import TOL, make_op, sample_points, set_filter, to_dev, to_host, torch

pytestmark = pytest.mark.gpu


def _dy(wl, inp):
    """A seeded loss gradient with the activations' dtype and distribution."""
    return W.make_inputs(wl, seed=wl.seed + 7).q


def _gpu_backward(op, inp, dy, spectrum=None, sbs=0):
    q, k, v, g = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), to_dev(dy)
    dq, dk, dv = op.backward(q, k, v, g, spectrum=spectrum, spectrum_batch_stride=sbs)
    torch().cuda.synchronize()
    st = op.status()
    assert st == H.OK, H.status_string(st)
    return to_host(dq), to_host(dk), to_host(dv)


def _as_f64(a):
    if a.dtype == np.uint16:
        return W.bf16_bits_to_f32(a).astype(np.float64)
    return a.astype(np.float64)


BWD = [
    ((32,), 2, 3, "f32"), ((256,), 1, 3, "bf16"),
    ((32, 16), 2, 2, "f32"), ((64, 64), 1, 3, "bf16"),
    ((256, 64), 1, 2, "f32"), ((128, 128), 2, 1, "bf16"), ((8, 256), 1, 2, "f32"),
    ((16, 16, 16), 2, 2, "f32"), ((32, 32, 64), 1, 2, "bf16"),
    ((16, 8, 32), 1, 2, "f32"), ((128, 128, 8), 1, 1, "f32"),
]


@pytest.mark.parametrize("dims,B,C,dt", BWD)
def test_backward_matches_oracle(dims, B, C, dt):
    wl = W.custom(dims, B, C, io_dtype=dt, seed=sum(dims) + 3 * B + C)
    inp = W.make_inputs(wl)
    dy = _dy(wl, inp)
    op = make_op(wl)
    set_filter(op, inp.filt)
    got = _gpu_backward(op, inp, dy)
    fwd_launches = {1: 1, 2: 1 if max(dims) <= 64 else 3, 3: 3}[len(dims)]
    if fwd_launches == 3:
        assert H.last_launch_count() % 6 == 0
    else:
        assert H.last_launch_count() == 2
    K = O.implicit_kernel(inp.filt, dims)
    S = O.spectrum_full(K, dims)
    want = O.backward_dft(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), _as_f64(dy), S, dims)
    for name, g, w in zip(("dq", "dk", "dv"), got, want):
        assert O.rel_l2(g, w) <= TOL[dt], name


def test_backward_full_size_sampled():
    """The 2D 256^2, B=2, C=128, bf16 workload (several waves per convolution):
    sampled outputs of all three gradients against direct sums."""
    wl = W.workload(2)
    inp = W.make_inputs(wl)
    dy = _dy(wl, inp)
    op = make_op(wl)
    set_filter(op, inp.filt)
    dq, dk, dv = _gpu_backward(op, inp, dy)
    assert H.last_launch_count() == 2 * H.plan_info(op.p)["launches"]
    chans = [0, 77, 127]
    pts = sample_points(wl, 10, seed=5, channels=chans)
    K = O.implicit_kernel(inp.filt, wl.dims, channels=chans)
    Kfull = np.zeros((wl.C,) + K.shape[1:])
    for j, c in enumerate(chans):
        Kfull[c] = K[j]
    q, k, v, g = inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), _as_f64(dy)
    w = O.conv_direct_at(np.ones_like(q), k, v, Kfull, wl.dims, pts)
    du = O.corr_direct_at(q * g, Kfull, wl.dims, pts)
    idx = [tuple(p) for p in pts]
    want_q = np.array([g[i] for i in idx]) * w
    want_k = np.array([v[i] for i in idx]) * du
    want_v = np.array([k[i] for i in idx]) * du
    for name, got, want in (("dq", dq, want_q), ("dk", dk, want_k), ("dv", dv, want_v)):
        assert O.rel_l2(np.array([got[i] for i in idx]), want) <= TOL["bf16"], name


def test_backward_per_sample_spectrum():
    dims = (32, 32, 16)
    wl = W.custom(dims, 2, 2, seed=41)
    inp = W.make_inputs(wl)
    dy = _dy(wl, inp)
    t = torch()
    rng = np.random.default_rng(3)
    Ks = [rng.standard_normal((2,) + tuple(2 * n - 1 for n in dims)) for _ in range(2)]
    op = make_op(wl)
    specs = []
    for Kb in Ks:
        op.import_spectrum(t.from_numpy(O.spectrum_half(Kb, dims).astype(np.complex64)))
        specs.append(op.spectrum.clone())
    both = t.cat(specs)
    got = _gpu_backward(op, inp, dy, spectrum=both, sbs=op.spec_bytes)
    q, k, v, g = inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), _as_f64(dy)
    for b in range(2):
        sl = slice(b, b + 1)
        want = O.backward_dft(q[sl], k[sl], v[sl], g[sl], O.spectrum_full(Ks[b], dims), dims)
        for name, gg, w in zip(("dq", "dk", "dv"), got, want):
            assert O.rel_l2(gg[sl], w) <= TOL["f32"], (b, name)


def test_backward_dq_equals_dy_times_forward_with_unit_gate():
    """On the GPU alone: with q = 1 the forward returns w = K * (k v), and the
    backward's dq must be dy w."""
    dims = (64, 64, 16)
    wl = W.custom(dims, 1, 2, seed=43)
    inp = W.make_inputs(wl)
    inp.q = np.ones_like(inp.q)
    dy = _dy(wl, inp)
    op = make_op(wl)
    set_filter(op, inp.filt)
    q, k, v, g = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), to_dev(dy)
    w = to_host(op(q, k, v))
    dq, _, _ = op.backward(q, k, v, g)
    dq = to_host(dq)
    assert np.allclose(dq, _as_f64(dy) * w, rtol=1e-5, atol=1e-6 * np.max(np.abs(dq)))
