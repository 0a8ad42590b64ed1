"""GPU parity of the kernel-value gradient
dK[c, t] = sum_b sum_i q[b,c,i] dy[b,c,i] (k v)[b,c,i - t] against the float64
oracle, on 1D, 2D and 3D grids, with several channel chunks, and sampled at the
benchmark size.  (Blog "Native multi-dimensional subquadratic operators via
input-dependent long convolutions", gradient sections: dK by correlation.)"""
import numpy as np
import pytest

from dimensional_long_convolution_b200 import hyena_nd as H
from dimensional_long_convolution_b200 import workloads as W
from oracle import hyena_nd_oracle as O

from gpu_util import TOL, make_op, to_dev, torch

pytestmark = pytest.mark.gpu


def _f64(a):
    return W.bf16_bits_to_f32(a).astype(np.float64) if a.dtype == np.uint16 else a.astype(np.float64)


def _gpu(wl, inp, dy):
    op = make_op(wl)
    dK = op.kernel_grad(to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), to_dev(dy))
    torch().cuda.synchronize()
    assert op.status() == H.OK
    return dK.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("dims,B,C,dt", [((32,), 2, 3, "f32"), ((256,), 1, 2, "bf16"), ((16, 32), 2, 2, "f32"),
                                         ((64, 64), 1, 2, "bf16"), ((8, 16, 8), 2, 2, "f32"),
                                         ((128, 128), 2, 53, "f32"),
                                         # 2D multi-pass grids: the row-pair / half-spectrum route, every
                                         # column-kernel geometry (n0 = 8 .. 256) and a single sample
                                         ((128, 256), 1, 2, "bf16"), ((256, 128), 3, 3, "f32"), ((8, 128), 2, 3, "f32"),
                                         ((256, 8), 2, 2, "f32"), ((16, 256), 1, 3, "f32"), ((32, 128), 2, 2, "bf16")])
def test_kernel_grad_matches_oracle(dims, B, C, dt):
    wl = W.custom(dims, B, C, io_dtype=dt, seed=5 + sum(dims))
    inp = W.make_inputs(wl, with_qkv=True)
    dy = W.make_inputs(wl, seed=wl.seed + 9).q
    got = _gpu(wl, inp, dy)
    want = O.kernel_grad_dft(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), _f64(dy), dims)
    assert got.shape == want.shape
    assert O.rel_l2(got, want) <= TOL[dt]


def test_kernel_grad_full_size_sampled():
    wl = W.workload(2)
    inp = W.make_inputs(wl)
    dy = W.make_inputs(wl, seed=wl.seed + 9).q
    got = _gpu(wl, inp, dy)
    rng = np.random.default_rng(4)
    pts = np.stack([rng.integers(0, wl.C, 12)] + [rng.integers(-(n - 1), n, 12) for n in wl.dims], axis=1)
    pts[0, 1:] = 0
    pts[1, 1:] = [n - 1 for n in wl.dims]
    pts[2, 1:] = [-(n - 1) for n in wl.dims]
    want = O.kernel_grad_at(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), _f64(dy), wl.dims, pts)
    gv = np.array([got[(p[0],) + tuple(int(t) + n - 1 for t, n in zip(p[1:], wl.dims))] for p in pts])
    assert O.rel_l2(gv, want) <= TOL["bf16"]
