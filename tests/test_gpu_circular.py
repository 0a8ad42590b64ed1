"""GPU parity of the circular (periodic) mode against the float64 oracle:
y[i] = q[i] sum_j u[j] Kper[(i - j) mod n] with Kper the filter at each
offset's representative in [-n/2, n/2); its backward and its kernel gradient on
the periodic grid.  (arXiv 2607.19378 summary, "Methodologie", boundary
handling: circular convolutions for periodic systems.)"""
import numpy as np
import pytest

from dimensional_long_convolution_b200 import hyena_nd as H
from dimensional_long_convolution_b200 import workloads as W
from oracle import hyena_nd_oracle as O

from gpu_util import TOL, set_filter, to_dev, to_host, torch

pytestmark = pytest.mark.gpu

CASES = [((32,), 2, 3, "f32"), ((256,), 1, 2, "bf16"), ((64, 64), 2, 2, "f32"), ((256, 128), 1, 2, "bf16"),
         ((16, 16, 32), 2, 2, "f32"), ((8, 16, 16), 1, 2, "f32"), ((128, 128, 8), 1, 1, "f32")]


def _f64(a):
    return W.bf16_bits_to_f32(a).astype(np.float64) if a.dtype == np.uint16 else a.astype(np.float64)


def _setup(dims, B, C, dt, seed):
    wl = W.custom(dims, B, C, io_dtype=dt, seed=seed)
    inp = W.make_inputs(wl)
    op = H.HyenaND(dims, B, C, dt, device="cuda", circular=1)
    set_filter(op, inp.filt)
    Kper = O.implicit_kernel_periodic(inp.filt, dims)
    return wl, inp, op, Kper


@pytest.mark.parametrize("dims,B,C,dt", CASES)
def test_circular_forward(dims, B, C, dt):
    wl, inp, op, Kper = _setup(dims, B, C, dt, 3 + sum(dims))
    y = op(to_dev(inp.q), to_dev(inp.k), to_dev(inp.v))
    torch().cuda.synchronize()
    assert op.status() == H.OK
    want = O.conv_circular(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), Kper, dims)
    assert O.rel_l2(to_host(y), want) <= TOL[dt]


@pytest.mark.parametrize("dims,B,C,dt", [CASES[0], CASES[2], CASES[3], CASES[4]])
def test_circular_backward(dims, B, C, dt):
    wl, inp, op, Kper = _setup(dims, B, C, dt, 7 + sum(dims))
    dy = W.make_inputs(wl, seed=wl.seed + 9).q
    dq, dk, dv = op.backward(to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), to_dev(dy))
    torch().cuda.synchronize()
    assert op.status() == H.OK
    S = O.spectrum_full(O.periodize_to_offsets(Kper, dims), dims)
    want = O.backward_dft(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), _f64(dy), S, dims)
    for name, g, w in zip(("dq", "dk", "dv"), (dq, dk, dv), want):
        assert O.rel_l2(to_host(g), w) <= TOL[dt], name


@pytest.mark.parametrize("dims,B,C,dt", [((32,), 2, 3, "f32"), ((16, 8), 2, 2, "f32"), ((8, 8, 16), 1, 2, "bf16")])
def test_circular_kernel_grad(dims, B, C, dt):
    wl, inp, op, _ = _setup(dims, B, C, dt, 11 + sum(dims))
    dy = W.make_inputs(wl, seed=wl.seed + 9).q
    dK = op.kernel_grad(to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), to_dev(dy))
    torch().cuda.synchronize()
    assert op.status() == H.OK
    assert tuple(dK.shape) == (C,) + dims
    want = O.kernel_grad_periodic_direct(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), _f64(dy), dims)
    assert O.rel_l2(dK.cpu().numpy().astype(np.float64), want) <= TOL[dt]
