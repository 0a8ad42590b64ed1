"""GPU parity of the per-sample filter call with FiLM conditioning against the
float64 oracle: sample b's spectrum from h_b = sin(gamma_b (W1 phi + b1) +
beta_b), then the batched forward and the backward with one spectrum per
sample.  (arXiv 2607.19378 summary, "Methodologie": kernels that depend on
the whole input sample through a control that modulates the coordinate
network feature-wise.)"""
import numpy as np
import pytest

from dimensional_long_convolution_b200 import hyena_nd as H
from dimensional_long_convolution_b200 import workloads as W
from oracle import hyena_nd_oracle as O

from gpu_util import TOL, to_dev, to_host, torch

pytestmark = pytest.mark.gpu


def _film(B, hidden, seed):
    rng = np.random.default_rng(seed)
    gamma = (1.0 + 0.5 * rng.standard_normal((B, hidden))).astype(np.float32)
    beta = (0.5 * rng.standard_normal((B, hidden))).astype(np.float32)
    return gamma, beta


def _f64(a):
    return W.bf16_bits_to_f32(a).astype(np.float64) if a.dtype == np.uint16 else a.astype(np.float64)


CASES = [((32,), 3, 2, "f32"), ((16, 32), 2, 3, "f32"), ((64, 64), 2, 2, "bf16"), ((256, 64), 2, 1, "f32"),
         ((16, 8, 32), 2, 2, "f32"), ((1024,), 2, 2, "f32")]


@pytest.mark.parametrize("dims,B,C,dt", CASES)
def test_film_spectra_and_forward(dims, B, C, dt):
    wl = W.custom(dims, B, C, io_dtype=dt, seed=sum(dims) + 5)
    inp = W.make_inputs(wl)
    f = inp.filt
    gamma, beta = _film(B, f.W1.shape[0], sum(dims))
    t = torch()
    op = H.HyenaND(dims, B, C, dt, device="cuda")
    specs = op.set_filter_film(*(t.from_numpy(a) for a in (f.W1, f.b1, f.W2, f.b2, f.alpha)), f.decay_scale,
                               t.from_numpy(gamma), t.from_numpy(beta), f.num_freqs)
    y = op(to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), spectrum=specs, spectrum_batch_stride=op.spec_bytes)
    t.cuda.synchronize()
    assert op.status() == H.OK
    got = to_host(y)
    q, k, v = inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v")
    per = op.spec_bytes // 8
    for b in range(B):
        Kb = O.implicit_kernel(f, dims, film=(gamma[b], beta[b]))
        # the exported spectrum of sample b equals the oracle's
        op.spectrum.copy_(specs[b * per:(b + 1) * per])
        assert O.rel_l2(to_host(op.export_spectrum()), O.spectrum_half(Kb, dims)) < 2e-5, b
        sl = slice(b, b + 1)
        want = O.conv_dft(q[sl], k[sl], v[sl], O.spectrum_full(Kb, dims), dims)
        assert O.rel_l2(got[sl], want) <= TOL[dt], b


def test_film_backward_per_sample():
    dims, B, C = (32, 16), 2, 3
    wl = W.custom(dims, B, C, seed=77)
    inp = W.make_inputs(wl)
    f = inp.filt
    gamma, beta = _film(B, f.W1.shape[0], 78)
    dy = W.make_inputs(wl, seed=79).q
    t = torch()
    op = H.HyenaND(dims, B, C, "f32", device="cuda")
    specs = op.set_filter_film(*(t.from_numpy(a) for a in (f.W1, f.b1, f.W2, f.b2, f.alpha)), f.decay_scale,
                               t.from_numpy(gamma), t.from_numpy(beta), f.num_freqs)
    dq, dk, dv = op.backward(to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), to_dev(dy), spectrum=specs,
                             spectrum_batch_stride=op.spec_bytes)
    t.cuda.synchronize()
    assert op.status() == H.OK
    q, k, v, g = inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), _f64(dy)
    for b in range(B):
        S = O.spectrum_full(O.implicit_kernel(f, dims, film=(gamma[b], beta[b])), dims)
        sl = slice(b, b + 1)
        want = O.backward_dft(q[sl], k[sl], v[sl], g[sl], S, dims)
        for name, gg, w in zip(("dq", "dk", "dv"), (dq, dk, dv), want):
            assert O.rel_l2(to_host(gg)[sl], w) <= TOL["f32"], (b, name)


def test_film_identity_matches_plain_filter():
    """gamma = 1, beta = 0 for every sample reproduces the shared filter call
    bit for bit (the same kernels run; the modulation is an exact fma)."""
    dims, B, C = (64, 64), 2, 4
    wl = W.custom(dims, B, C, seed=81)
    inp = W.make_inputs(wl, with_qkv=False)
    f = inp.filt
    H_ = f.W1.shape[0]
    t = torch()
    op = H.HyenaND(dims, B, C, "f32", device="cuda")
    w = [t.from_numpy(a) for a in (f.W1, f.b1, f.W2, f.b2, f.alpha)]
    specs = op.set_filter_film(*w, f.decay_scale, t.ones(B, H_), t.zeros(B, H_), f.num_freqs)
    op.set_filter(*w, f.decay_scale, f.num_freqs)
    t.cuda.synchronize()
    per = op.spec_bytes // 8
    for b in range(B):
        assert t.equal(specs[b * per:(b + 1) * per], op.spectrum), b
