"""The index-checked build (libhyena_nd_bounds.so, HYENA_ND_BOUNDS): every
kernel access to a caller buffer or to shared memory is checked against the
call's registered buffers and the CTA's dynamic shared memory; a violation is
recorded as HYENA_ND_ERR_DEVICE_BOUNDS and the access is redirected to a
dummy location instead of touching memory.  This stands in for a memory
sanitizer.

One small case per tier and per entry point runs on the checked build in a
child process (the binding loads one library per process); each must leave
the status word clean and match the float64 oracle within the parity
tolerances.  (HyenaND blog, section "HyenaND", output equation; arXiv
2607.19378 summary, "Methodologie": zero padding to twice the grid.)"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BOUNDS_LIB = os.path.join(ROOT, "dimensional_long_convolution_b200", "libhyena_nd_bounds.so")

# (dims, B, C, dtype): 1D rows, long 1D, fused 2D, multi-pass 2D, multi-pass
# 3D, the 2-CTA 128 x 128 slab pair
CONV = [((64,), 2, 3, "f32"), ((1024,), 1, 2, "f32"), ((32, 64), 2, 2, "bf16"), ((128, 256), 1, 2, "f32"),
        ((16, 32, 64), 1, 2, "f32"), ((128, 128, 8), 1, 1, "f32")]
BWD = [((32, 32), 1, 2, "f32"), ((64, 128), 1, 2, "f32"), ((8, 16, 32), 1, 2, "f32")]
KGRAD = [((32, 16), 2, 2, "f32"), ((64, 128), 2, 2, "f32"), ((8, 8, 16), 1, 2, "f32"), ((512,), 1, 2, "f32")]
# a three-level long 1D grid: 2^19 points split 128 x 64 x 64, odd C
PLANE = [(1 << 18, 1, 3, "f32")]


def _child() -> None:
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from dimensional_long_convolution_b200 import hyena_nd as H
    H.load(BOUNDS_LIB)
    from dimensional_long_convolution_b200 import workloads as W
    from oracle import hyena_nd_oracle as O
    from gpu_util import make_op, run, set_filter, to_dev, to_host, torch
    t = torch()
    out = []

    def f64(a):
        return W.bf16_bits_to_f32(a).astype(np.float64) if a.dtype == np.uint16 else a.astype(np.float64)

    for dims, B, C, dt in CONV:
        wl = W.custom(dims, B, C, io_dtype=dt, seed=3 + sum(dims))
        inp = W.make_inputs(wl)
        got, op = run(inp)                          # asserts a clean status word
        out.append({"what": "conv %s" % (dims,), "dt": dt, "err": O.rel_l2(got, O.reference_output(inp)),
                    "status": int(H.device_status(op.ws.data_ptr(), op._stream()))})
        # the no-allocation entry point on the same problem
        q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
        y = t.empty_like(q)
        st = H.fftconv_batched_static(op.p, q.data_ptr(), k.data_ptr(), v.data_ptr(), op.spectrum.data_ptr(), 0,
                                      y.data_ptr(), op._stream())
        t.cuda.synchronize()
        out.append({"what": "static %s" % (dims,), "dt": dt, "call": int(st),
                    "err": O.rel_l2(to_host(y), O.reference_output(inp)),
                    "status": int(H.device_status(0, op._stream()))})
        # spectrum export back to the oracle's natural order
        nat = to_host(op.export_spectrum())
        want = O.spectrum_half(O.implicit_kernel(inp.filt, dims), dims) if np.prod(dims) <= 65536 else None
        if want is not None:
            out.append({"what": "export %s" % (dims,), "dt": "f32", "err": O.rel_l2(nat, want),
                        "status": int(H.device_status(op.ws.data_ptr(), op._stream()))})
    # a three-level long 1D split (five passes, the channel-pair center
    # pass), sampled against direct sums
    from gpu_util import sample_points
    for n, B, C, dt in PLANE:
        wl = W.custom((n,), B, C, io_dtype=dt, seed=29)
        inp = W.make_inputs(wl)
        got, op = run(inp)
        chans = sorted({0, C - 1})
        pts = sample_points(wl, 8, seed=5, channels=chans)
        K = np.zeros((C, 2 * n - 1))
        Kc = O.implicit_kernel(inp.filt, (n,), channels=chans)
        for j, c in enumerate(chans):
            K[c] = Kc[j]
        want = O.conv_direct_at(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), K, (n,), pts)
        gv = np.array([got[tuple(p)] for p in pts])
        out.append({"what": "long 1D %d" % n, "dt": dt, "err": O.rel_l2(gv, want),
                    "status": int(H.device_status(op.ws.data_ptr(), op._stream()))})
    for dims, B, C, dt in BWD:
        wl = W.custom(dims, B, C, io_dtype=dt, seed=11 + sum(dims))
        inp = W.make_inputs(wl)
        dy = W.make_inputs(wl, seed=wl.seed + 7).q
        op = make_op(wl)
        set_filter(op, inp.filt)
        g = op.backward(to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), to_dev(dy))
        t.cuda.synchronize()
        S = O.spectrum_full(O.implicit_kernel(inp.filt, dims), dims)
        want = O.backward_dft(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), f64(dy), S, dims)
        err = max(O.rel_l2(to_host(a), b) for a, b in zip(g, want))
        out.append({"what": "backward %s" % (dims,), "dt": dt, "err": err,
                    "status": int(H.device_status(op.ws.data_ptr(), op._stream()))})
    for dims, B, C, dt in KGRAD:
        wl = W.custom(dims, B, C, io_dtype=dt, seed=19 + sum(dims))
        inp = W.make_inputs(wl)
        dy = W.make_inputs(wl, seed=wl.seed + 9).q
        op = make_op(wl)
        dK = op.kernel_grad(to_dev(inp.q), to_dev(inp.k), to_dev(inp.v), to_dev(dy))
        t.cuda.synchronize()
        want = O.kernel_grad_dft(inp.as_f64("q"), inp.as_f64("k"), inp.as_f64("v"), f64(dy), dims)
        out.append({"what": "kernel_grad %s" % (dims,), "dt": dt,
                    "err": O.rel_l2(dK.cpu().numpy().astype(np.float64), want),
                    "status": int(H.device_status(op.ws.data_ptr(), op._stream()))})
    print("RESULTS " + json.dumps(out))


@pytest.mark.gpu
def test_checked_build_is_clean_and_matches_the_oracle():
    if not os.path.exists(BOUNDS_LIB):
        from dimensional_long_convolution_b200 import build as B
        B.build(bounds=True)
    r = subprocess.run([sys.executable, os.path.abspath(__file__), "child"], capture_output=True, text=True,
                       timeout=1200)
    assert r.returncode == 0, r.stderr[-3000:]
    line = [l for l in r.stdout.splitlines() if l.startswith("RESULTS ")]
    assert line, r.stdout[-2000:]
    res = json.loads(line[-1][len("RESULTS "):])
    tol = {"f32": 1e-4, "bf16": 1e-2}
    for e in res:
        assert e["status"] == 0, e            # no bounds violation, no timeout
        assert e.get("call", 0) == 0, e
        assert e["err"] <= tol[e["dt"]], e


if __name__ == "__main__" and len(sys.argv) > 1 and sys.argv[1] == "child":
    _child()
