"""Shared helpers for the GPU parity tests: move seeded inputs to the device,
run the library through its C ABI (ctypes binding), bring results back."""
import numpy as np

from dimensional_long_convolution_b200 import hyena_nd as H
from dimensional_long_convolution_b200 import workloads as W

# Tolerances on the relative L2 error against the float64 oracle, as the task
# states them: fp32 activations 1e-4, bf16 activations (fp32 compute) 1e-2.
TOL = {"f32": 1e-4, "bf16": 1e-2}


def torch():
    import torch as _t
    return _t


def to_dev(a: np.ndarray):
    t = torch()
    if a.dtype == np.uint16:
        return t.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(t.bfloat16)
    return t.from_numpy(np.ascontiguousarray(a)).cuda()


def to_host(x) -> np.ndarray:
    t = torch()
    if x.dtype == t.bfloat16:
        return x.float().cpu().numpy().astype(np.float64)
    if x.dtype == t.complex64:
        return x.cpu().numpy().astype(np.complex128)
    return x.cpu().numpy().astype(np.float64)


def make_op(wl):
    return H.HyenaND(wl.dims, wl.B, wl.C, wl.io_dtype, device="cuda")


def set_filter(op, filt):
    t = torch()
    op.set_filter(t.from_numpy(filt.W1), t.from_numpy(filt.b1), t.from_numpy(filt.W2), t.from_numpy(filt.b2),
                  t.from_numpy(filt.alpha), filt.decay_scale, filt.num_freqs)


def run(inp, natural_spectrum=None, op=None, sbs=0, spectrum=None):
    """y (float64, host) from the GPU path for seeded inputs ``inp``.  The
    spectrum comes from the library's filter call unless a natural-order one
    is given."""
    t = torch()
    wl = inp.wl
    if op is None:
        op = make_op(wl)
        if natural_spectrum is None:
            set_filter(op, inp.filt)
        else:
            op.import_spectrum(t.from_numpy(np.ascontiguousarray(natural_spectrum.astype(np.complex64))))
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    y = op(q, k, v, spectrum=spectrum, spectrum_batch_stride=sbs)
    t.cuda.synchronize()
    st = op.status()
    assert st == H.OK, H.status_string(st)
    return to_host(y), op


def sample_points(wl, m, seed=0, channels=None):
    rng = np.random.default_rng(seed)
    b = rng.integers(0, wl.B, m)
    c = rng.integers(0, wl.C, m) if channels is None else rng.choice(np.asarray(channels), m)
    idx = [rng.integers(0, n, m) for n in wl.dims]
    pts = np.stack([b, c] + idx, axis=1)
    # always include the corners of the crop window
    pts[0, 2:] = 0
    pts[1, 2:] = np.array(wl.dims) - 1
    return pts
