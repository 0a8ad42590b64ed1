"""Thin ctypes binding of libhyena_nd.so (the C ABI in include/hyena_nd.h).

Argument marshalling only: every step of the convolution runs in the CUDA
kernels of the shared library.  The functions carry the C names without the
``hyena_nd_`` prefix and take raw integers (device pointers, byte counts,
stream handles).  ``HyenaND`` below wraps them for torch tensors: torch
provides device memory and the current stream, nothing else.

Importing this module never falls back to anything: if the shared library is
missing or fails to load, ``load()`` raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhyena_nd.so")

OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED = 2
ERR_MISALIGNED = 3
ERR_WORKSPACE_TOO_SMALL = 4
ERR_CUDA = 5
ERR_DEVICE_TIMEOUT = 6
ERR_DEVICE_BOUNDS = 7

F32 = 0
BF16 = 1

# calls that use a workspace (hyena_nd_workspace_bytes_for)
CALL_ALL = 0
CALL_CONV = 1
CALL_FILTER = 2
CALL_KERNEL_GRAD = 3

EXPORTED = (
    "hyena_nd_spectrum_bytes",
    "hyena_nd_workspace_bytes",
    "hyena_nd_workspace_bytes_for",
    "hyena_nd_workspace_init",
    "hyena_nd_filter_spectrum",
    "hyena_nd_filter_spectrum_film",
    "hyena_nd_fftconv",
    "hyena_nd_fftconv_batched",
    "hyena_nd_fftconv_backward",
    "hyena_nd_kernel_grad",
    "hyena_nd_spectrum_export",
    "hyena_nd_spectrum_import",
    "hyena_nd_device_status",
    "hyena_nd_debug_bounded_wait",
    "hyena_nd_status_string",
    "hyena_nd_last_launch_count",
    "hyena_nd_fftconv_batched_static",
    "hyena_nd_plan_info_get",
)

TIERS = {0: "rows_1d", 1: "fused_2d", 2: "multi_2d", 3: "multi_3d", 4: "long_1d"}

STATIC_SCRATCH_BYTES = 16 << 20


class PlanInfo(ctypes.Structure):
    _fields_ = [
        ("tier", ctypes.c_int),
        ("wave", ctypes.c_int64),
        ("waves", ctypes.c_int64),
        ("launches", ctypes.c_int),
        ("split_levels", ctypes.c_int),
        ("split", ctypes.c_int * 3),
        ("filter_chunk", ctypes.c_int),
        ("kgrad_chunk", ctypes.c_int),
        ("workspace_bytes", ctypes.c_size_t),
        ("spectrum_bytes", ctypes.c_size_t),
        ("streams", ctypes.c_int),
    ]


class Problem(ctypes.Structure):
    _fields_ = [
        ("ndim", ctypes.c_int),
        ("n", ctypes.c_int64 * 3),
        ("B", ctypes.c_int64),
        ("C", ctypes.c_int64),
        ("io_dtype", ctypes.c_int),
        ("circular", ctypes.c_int),
    ]


class Filter(ctypes.Structure):
    _fields_ = [
        ("num_freqs", ctypes.c_int),
        ("hidden", ctypes.c_int),
        ("W1", ctypes.c_void_p),
        ("b1", ctypes.c_void_p),
        ("W2", ctypes.c_void_p),
        ("b2", ctypes.c_void_p),
        ("alpha", ctypes.c_void_p),
        ("decay_scale", ctypes.c_float),
        ("window", ctypes.c_int),
    ]


class HyenaNDError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__("%s failed: %s" % (what, status_string(code)))


_lib: Optional[ctypes.CDLL] = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the shared library (once).  Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError("libhyena_nd.so not built at %s (run python -m dimensional_long_convolution_b200.build)" % path)
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER(Problem)
    vp, sz, i64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int64
    sigs = {
        "hyena_nd_spectrum_bytes": (sz, [P]),
        "hyena_nd_workspace_bytes": (sz, [P]),
        "hyena_nd_workspace_bytes_for": (ctypes.c_size_t, [P, ctypes.c_int]),
        "hyena_nd_workspace_init": (ctypes.c_int, [vp, sz, vp]),
        "hyena_nd_filter_spectrum": (ctypes.c_int, [P, ctypes.POINTER(Filter), vp, vp, sz, vp]),
        "hyena_nd_filter_spectrum_film": (ctypes.c_int, [P, ctypes.POINTER(Filter), vp, vp, vp, i64, vp, sz, vp]),
        "hyena_nd_fftconv": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, sz, vp]),
        "hyena_nd_fftconv_batched": (ctypes.c_int, [P, vp, vp, vp, vp, i64, vp, vp, sz, vp]),
        "hyena_nd_fftconv_backward": (ctypes.c_int, [P, vp, vp, vp, vp, i64, vp, vp, vp, vp, vp, sz, vp]),
        "hyena_nd_kernel_grad": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, sz, vp]),
        "hyena_nd_spectrum_export": (ctypes.c_int, [P, vp, vp, vp]),
        "hyena_nd_spectrum_import": (ctypes.c_int, [P, vp, vp, vp]),
        "hyena_nd_device_status": (ctypes.c_int, [vp, vp]),
        "hyena_nd_debug_bounded_wait": (ctypes.c_int, [vp, sz, ctypes.c_int, vp]),
        "hyena_nd_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "hyena_nd_last_launch_count": (ctypes.c_int, []),
        "hyena_nd_fftconv_batched_static": (ctypes.c_int, [P, vp, vp, vp, vp, i64, vp, vp]),
        "hyena_nd_plan_info_get": (ctypes.c_int, [P, ctypes.POINTER(PlanInfo)]),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def problem(dims: Sequence[int], B: int, C: int, io_dtype: int = F32, circular: int = 0) -> Problem:
    p = Problem()
    p.ndim = len(dims)
    for i in range(3):
        p.n[i] = int(dims[i]) if i < len(dims) else 0
    p.B, p.C, p.io_dtype, p.circular = int(B), int(C), int(io_dtype), int(circular)
    return p


# ------------------------------------------------------------ raw C calls
def spectrum_bytes(p: Problem) -> int:
    return int(load().hyena_nd_spectrum_bytes(ctypes.byref(p)))


def workspace_bytes(p: Problem) -> int:
    return int(load().hyena_nd_workspace_bytes(ctypes.byref(p)))


def workspace_bytes_for(p: Problem, call: int) -> int:
    return int(load().hyena_nd_workspace_bytes_for(ctypes.byref(p), int(call)))


def workspace_init(ws: int, ws_bytes: int, stream: int = 0) -> int:
    return load().hyena_nd_workspace_init(ws, ws_bytes, stream)


def filter_spectrum(p: Problem, f: Filter, spectrum: int, ws: int, ws_bytes: int, stream: int = 0) -> int:
    return load().hyena_nd_filter_spectrum(ctypes.byref(p), ctypes.byref(f), spectrum, ws, ws_bytes, stream)


def filter_spectrum_film(p: Problem, f: Filter, gamma: int, beta: int, spectrum: int, spectrum_batch_stride: int,
                         ws: int, ws_bytes: int, stream: int = 0) -> int:
    return load().hyena_nd_filter_spectrum_film(ctypes.byref(p), ctypes.byref(f), gamma, beta, spectrum,
                                                spectrum_batch_stride, ws, ws_bytes, stream)


def fftconv(p: Problem, q: int, k: int, v: int, spectrum_c: int, y: int, ws: int, ws_bytes: int,
            stream: int = 0) -> int:
    return load().hyena_nd_fftconv(ctypes.byref(p), q, k, v, spectrum_c, y, ws, ws_bytes, stream)


def fftconv_batched(p: Problem, q: int, k: int, v: int, spectrum: int, spectrum_batch_stride: int, y: int,
                    ws: int, ws_bytes: int, stream: int = 0) -> int:
    return load().hyena_nd_fftconv_batched(ctypes.byref(p), q, k, v, spectrum, spectrum_batch_stride, y, ws,
                                           ws_bytes, stream)


def fftconv_batched_static(p: Problem, q: int, k: int, v: int, spectrum: int, spectrum_batch_stride: int,
                           y: int, stream: int = 0) -> int:
    """The batched call without a workspace argument: its scratch is a fixed
    16 MiB array inside the library (for callers that cannot allocate)."""
    return load().hyena_nd_fftconv_batched_static(ctypes.byref(p), q, k, v, spectrum, spectrum_batch_stride, y,
                                                  stream)


def spectrum_export(p: Problem, spectrum: int, natural: int, stream: int = 0) -> int:
    return load().hyena_nd_spectrum_export(ctypes.byref(p), spectrum, natural, stream)


def spectrum_import(p: Problem, natural: int, spectrum: int, stream: int = 0) -> int:
    return load().hyena_nd_spectrum_import(ctypes.byref(p), natural, spectrum, stream)


def device_status(ws: int, stream: int = 0) -> int:
    return load().hyena_nd_device_status(ws, stream)


def debug_bounded_wait(ws: int, ws_bytes: int, limit_us: int, stream: int = 0) -> int:
    return load().hyena_nd_debug_bounded_wait(ws, ws_bytes, int(limit_us), stream)


def fftconv_backward(p: Problem, q: int, k: int, v: int, spectrum: int, spectrum_batch_stride: int, dy: int,
                     dq: int, dk: int, dv: int, ws: int, ws_bytes: int, stream: int = 0) -> int:
    return load().hyena_nd_fftconv_backward(ctypes.byref(p), q, k, v, spectrum, int(spectrum_batch_stride), dy,
                                            dq, dk, dv, ws, ws_bytes, stream)


def kernel_grad(p: Problem, q: int, k: int, v: int, dy: int, dK: int, ws: int, ws_bytes: int,
                stream: int = 0) -> int:
    return load().hyena_nd_kernel_grad(ctypes.byref(p), q, k, v, dy, dK, ws, ws_bytes, stream)


def plan_info(p: Problem) -> dict:
    """The execution plan of a problem (host only): tier, waves, launches per
    convolution, long-1D split, chunk sizes and buffer sizes."""
    info = PlanInfo()
    check(load().hyena_nd_plan_info_get(ctypes.byref(p), ctypes.byref(info)), "plan_info")
    return {"tier": TIERS.get(info.tier, str(info.tier)), "wave": info.wave, "waves": info.waves,
            "launches": info.launches, "split_levels": info.split_levels, "split": list(info.split),
            "filter_chunk": info.filter_chunk, "kgrad_chunk": info.kgrad_chunk,
            "workspace_bytes": info.workspace_bytes, "spectrum_bytes": info.spectrum_bytes,
            "streams": info.streams}


def status_string(code: int) -> str:
    return load().hyena_nd_status_string(int(code)).decode()


def last_launch_count() -> int:
    return int(load().hyena_nd_last_launch_count())


def check(code: int, what: str) -> None:
    if code != OK:
        raise HyenaNDError(code, what)


# ------------------------------------------------------------ torch wrapper
class HyenaND:
    """One problem shape bound to a device: owns the spectrum and workspace
    tensors (allocated by torch) and calls the C ABI on the current stream."""

    def __init__(self, dims: Sequence[int], B: int, C: int, io_dtype: str = "f32", device=None, circular: int = 0):
        import torch

        self.torch = torch
        self.dims = tuple(int(d) for d in dims)
        self.B, self.C = int(B), int(C)
        self.io_dtype = io_dtype
        self.tdtype = torch.bfloat16 if io_dtype == "bf16" else torch.float32
        self.circular = int(circular)
        self.p = problem(self.dims, B, C, BF16 if io_dtype == "bf16" else F32, circular=self.circular)
        dev = torch.device(device if device is not None else "cuda")
        if dev.type == "cuda" and dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
        self.device = dev
        nbytes = workspace_bytes(self.p)
        if nbytes == 0:
            raise HyenaNDError(ERR_UNSUPPORTED, "workspace_bytes")
        self.ws_bytes = nbytes
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        self.spec_bytes = spectrum_bytes(self.p)
        self.spectrum = torch.empty(self.spec_bytes // 8, dtype=torch.complex64, device=self.device)
        check(workspace_init(self.ws.data_ptr(), nbytes, self._stream()), "workspace_init")

    def _stream(self) -> int:
        return int(self.torch.cuda.current_stream(self.device).cuda_stream)

    def natural_shape(self):
        P = [2 * n for n in self.dims]
        return (self.C,) + tuple(P[:-1]) + (self.dims[-1] + 1,)

    def set_filter(self, W1, b1, W2, b2, alpha, decay_scale: float, num_freqs: int = 8, window: int = 0) -> None:
        t = [x.to(self.device, self.torch.float32).contiguous() for x in (W1, b1, W2, b2, alpha)]
        self._filter_params = t        # keep alive until the call has run
        f = Filter()
        f.num_freqs = int(num_freqs)
        f.hidden = int(t[0].shape[0])
        f.W1, f.b1, f.W2, f.b2, f.alpha = (x.data_ptr() for x in t)
        f.decay_scale = float(decay_scale)
        f.window = int(window)
        check(filter_spectrum(self.p, f, self.spectrum.data_ptr(), self.ws.data_ptr(), self.ws_bytes,
                              self._stream()), "filter_spectrum")

    def set_filter_film(self, W1, b1, W2, b2, alpha, decay_scale: float, gamma, beta, num_freqs: int = 8,
                        window: int = 0):
        """Per-sample spectra from one filter network under per-sample FiLM
        modulation gamma, beta [B, hidden]: returns a complex64 tensor holding
        B spectra back to back (the stride to pass to the convolution calls is
        ``self.spec_bytes``)."""
        t = [x.to(self.device, self.torch.float32).contiguous() for x in (W1, b1, W2, b2, alpha, gamma, beta)]
        f = Filter()
        f.num_freqs = int(num_freqs)
        f.hidden = int(t[0].shape[0])
        f.W1, f.b1, f.W2, f.b2, f.alpha = (x.data_ptr() for x in t[:5])
        f.decay_scale = float(decay_scale)
        f.window = int(window)
        if tuple(t[5].shape) != (self.B, f.hidden) or tuple(t[6].shape) != (self.B, f.hidden):
            raise ValueError("gamma and beta must be [B, hidden]")
        out = self.torch.empty(self.B * (self.spec_bytes // 8), dtype=self.torch.complex64, device=self.device)
        check(filter_spectrum_film(self.p, f, t[5].data_ptr(), t[6].data_ptr(), out.data_ptr(), self.spec_bytes,
                                   self.ws.data_ptr(), self.ws_bytes, self._stream()), "filter_spectrum_film")
        self._film_params = t
        return out

    def import_spectrum(self, natural) -> None:
        nat = natural.to(self.device, self.torch.complex64).contiguous()
        check(spectrum_import(self.p, nat.data_ptr(), self.spectrum.data_ptr(), self._stream()), "spectrum_import")
        self._import_keep = nat

    def export_spectrum(self):
        out = self.torch.empty(self.natural_shape(), dtype=self.torch.complex64, device=self.device)
        check(spectrum_export(self.p, self.spectrum.data_ptr(), out.data_ptr(), self._stream()), "spectrum_export")
        return out

    def __call__(self, q, k, v, y=None, spectrum=None, spectrum_batch_stride: int = 0):
        for t in (q, k, v):
            if t.dtype != self.tdtype or not t.is_contiguous() or t.device != self.device:
                raise ValueError("q, k, v must be contiguous %s tensors on %s" % (self.tdtype, self.device))
        if y is None:
            y = self.torch.empty_like(q)
        spec = self.spectrum if spectrum is None else spectrum
        check(fftconv_batched(self.p, q.data_ptr(), k.data_ptr(), v.data_ptr(), spec.data_ptr(),
                              int(spectrum_batch_stride), y.data_ptr(), self.ws.data_ptr(), self.ws_bytes,
                              self._stream()), "fftconv_batched")
        return y

    def backward(self, q, k, v, dy, spectrum=None, spectrum_batch_stride: int = 0):
        """(dq, dk, dv) for the loss gradient dy of __call__'s output."""
        for t in (q, k, v, dy):
            if t.dtype != self.tdtype or not t.is_contiguous() or t.device != self.device:
                raise ValueError("q, k, v, dy must be contiguous %s tensors on %s" % (self.tdtype, self.device))
        dq, dk, dv = (self.torch.empty_like(q) for _ in range(3))
        spec = self.spectrum if spectrum is None else spectrum
        check(fftconv_backward(self.p, q.data_ptr(), k.data_ptr(), v.data_ptr(), spec.data_ptr(),
                               int(spectrum_batch_stride), dy.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                               dv.data_ptr(), self.ws.data_ptr(), self.ws_bytes, self._stream()), "fftconv_backward")
        return dq, dk, dv

    def kernel_grad(self, q, k, v, dy):
        """dK (float32): the gradient of the loss with respect to the kernel
        values, for the loss gradient dy of __call__'s output; [C, 2n-1, ...]
        on the linear offsets, [C, n...] on the periodic grid when circular."""
        for t in (q, k, v, dy):
            if t.dtype != self.tdtype or not t.is_contiguous() or t.device != self.device:
                raise ValueError("q, k, v, dy must be contiguous %s tensors on %s" % (self.tdtype, self.device))
        shape = tuple(self.dims) if self.circular else tuple(2 * n - 1 for n in self.dims)
        dK = self.torch.empty((self.C,) + shape, dtype=self.torch.float32, device=self.device)
        check(kernel_grad(self.p, q.data_ptr(), k.data_ptr(), v.data_ptr(), dy.data_ptr(), dK.data_ptr(),
                          self.ws.data_ptr(), self.ws_bytes, self._stream()), "kernel_grad")
        return dK

    def status(self) -> int:
        return device_status(self.ws.data_ptr(), self._stream())
