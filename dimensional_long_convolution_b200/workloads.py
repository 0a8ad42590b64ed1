"""Seeded synthetic workloads for the gated nD FFT long convolution.

This module only *generates inputs*: the five benchmark grids, the random
activations q, k, v and the random parameters of the implicit filter MLP.  It
holds none of the convolution's arithmetic, so both the CUDA path's tests and
the float64 CPU oracle can draw identical inputs from it.

Workload shapes follow the benchmark spec of the HyenaND pages
("Native Multi-Dimensional Subquadratic Operators via Input Dependent Long
Convolutions", Methodologie / Implementation sections): native 2D image grids
and 3D volumes, zero-padded (linear) convolution, an implicit per-channel
filter built from sin/cos Fourier features of the offset, a sine-activated MLP
and an exponential decay window.

Random draw order (numpy PCG64, ``np.random.default_rng(seed)``):
q, k, v (standard normal, scaled), W1, b1, W2, b2 (normal with variance
1/fan_in), then -- only for the smooth-volume workload -- the parameters of 4
random 3D sinusoids per tensor (q, k, v in that order).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional, Tuple

import numpy as np

NUM_FREQS = 8      # Fourier features per axis: sin/cos of pi*m*t/n, m = 1..8
HIDDEN = 64        # width of the filter MLP's hidden layer


@dataclass(frozen=True)
class Workload:
    name: str
    dims: Tuple[int, ...]        # native grid (n1, ..., nd), last axis contiguous
    B: int
    C: int
    io_dtype: str                # "f32" or "bf16"
    input_scale: float = 1.0     # q, k, v ~ input_scale * N(0, 1)
    smooth: bool = False         # add 4 random low-frequency 3D sinusoids
    seed: int = 1234

    @property
    def ndim(self) -> int:
        return len(self.dims)

    @property
    def voxels(self) -> int:
        return int(np.prod(self.dims))

    @property
    def decay_scale(self) -> float:
        # exp(-alpha_c * ||t|| / s) with s the grid side of the workload
        return float(self.dims[0])

    @property
    def padded(self) -> Tuple[int, ...]:
        return tuple(2 * n for n in self.dims)


# The five grids of the benchmark suite (image token grid, high-resolution
# image, volume, large smooth volume), in the order the suite lists them.
WORKLOADS = (
    Workload("grid2d_32_b1_c4_f32", (32, 32), 1, 4, "f32", seed=1234),
    Workload("grid2d_64_b8_c256_f32", (64, 64), 8, 256, "f32", seed=1235),
    Workload("grid2d_256_b2_c128_bf16", (256, 256), 2, 128, "bf16", input_scale=0.5, seed=1236),
    Workload("grid3d_64_b2_c64_f32", (64, 64, 64), 2, 64, "f32", seed=1237),
    Workload("grid3d_128_b1_c32_bf16", (128, 128, 128), 1, 32, "bf16", smooth=True, seed=1238),
)


# Long 1D sequences (the pages' long-context class: about a million and about
# ten million tokens), measured beside the suite as extra lines.
EXTRA = (
    Workload("seq1d_1m_b1_c64_bf16", (1 << 20,), 1, 64, "bf16", input_scale=0.5, seed=1240),
    Workload("seq1d_8m_b1_c8_f32", (1 << 23,), 1, 8, "f32", seed=1241),
)


def workload(i_or_name) -> Workload:
    if isinstance(i_or_name, int):
        return WORKLOADS[i_or_name]
    for w in WORKLOADS + EXTRA:
        if w.name == i_or_name:
            return w
    raise KeyError(i_or_name)


def custom(dims, B, C, io_dtype="f32", seed=7, input_scale=1.0, smooth=False) -> Workload:
    """A small ad-hoc workload (test sizes: d = 1, 2, 3, non-square grids)."""
    return Workload("custom_" + "x".join(map(str, dims)), tuple(int(d) for d in dims), int(B), int(C),
                    io_dtype, input_scale=input_scale, smooth=smooth, seed=seed)


# ---------------------------------------------------------------- bf16 helpers
def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round-to-nearest-even."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    bits = f.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    rounded = ((bits + 0x7FFF + lsb) >> 16).astype(np.uint16)
    return rounded


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass
class FilterParams:
    """Parameters of the implicit filter MLP (fp32, exactly what the GPU sees)."""
    W1: np.ndarray      # [HIDDEN, 2*NUM_FREQS*d]
    b1: np.ndarray      # [HIDDEN]
    W2: np.ndarray      # [C, HIDDEN]
    b2: np.ndarray      # [C]
    alpha: np.ndarray   # [C]   decay rates, log-spaced in [0.5, 5]
    decay_scale: float
    num_freqs: int = NUM_FREQS
    hidden: int = HIDDEN


@dataclass
class Inputs:
    wl: Workload
    q: np.ndarray            # device-visible values: float32 array, or uint16 bf16 bits
    k: np.ndarray
    v: np.ndarray
    filt: FilterParams
    extra: dict = field(default_factory=dict)

    def as_f64(self, name: str) -> np.ndarray:
        """The exact values the GPU sees, widened to float64."""
        a = getattr(self, name)
        if a.dtype == np.uint16:
            return bf16_bits_to_f32(a).astype(np.float64)
        return a.astype(np.float64)


def _smooth_field(rng, dims) -> np.ndarray:
    """Sum of 4 random sinusoids a*sin(2*pi*f.x/n + phi) over the grid."""
    d = len(dims)
    f = rng.integers(1, 4, size=(4, d))
    a = rng.uniform(0.5, 1.0, size=4)
    phi = rng.uniform(0.0, 2.0 * np.pi, size=4)
    grids = np.meshgrid(*[np.arange(n, dtype=np.float64) / n for n in dims], indexing="ij")
    out = np.zeros(dims, dtype=np.float64)
    for m in range(4):
        arg = sum(2.0 * np.pi * f[m, ax] * grids[ax] for ax in range(d)) + phi[m]
        out += a[m] * np.sin(arg)
    return out


def make_filter_params(rng, ndim: int, C: int, decay_scale: float) -> FilterParams:
    fin = 2 * NUM_FREQS * ndim
    W1 = rng.normal(0.0, 1.0 / np.sqrt(fin), size=(HIDDEN, fin)).astype(np.float32)
    b1 = rng.normal(0.0, 1.0 / np.sqrt(fin), size=(HIDDEN,)).astype(np.float32)
    W2 = rng.normal(0.0, 1.0 / np.sqrt(HIDDEN), size=(C, HIDDEN)).astype(np.float32)
    b2 = rng.normal(0.0, 1.0 / np.sqrt(HIDDEN), size=(C,)).astype(np.float32)
    if C > 1:
        alpha = 0.5 * 10.0 ** (np.arange(C, dtype=np.float64) / (C - 1))
    else:
        alpha = np.array([0.5])
    return FilterParams(W1, b1, W2, b2, alpha.astype(np.float32), float(decay_scale))


def make_inputs(wl: Workload, seed: Optional[int] = None, with_qkv: bool = True) -> Inputs:
    """Draw q, k, v and the filter parameters for workload ``wl``."""
    rng = np.random.default_rng(wl.seed if seed is None else seed)
    shape = (wl.B, wl.C) + tuple(wl.dims)
    acts = []
    for _ in range(3):
        if with_qkv:
            acts.append(rng.standard_normal(size=shape) * wl.input_scale)
        else:
            acts.append(None)
    filt = make_filter_params(rng, wl.ndim, wl.C, wl.decay_scale)
    if wl.smooth and with_qkv:
        for i in range(3):
            acts[i] = acts[i] + _smooth_field(rng, wl.dims)[None, None]
    out = []
    for a in acts:
        if a is None:
            out.append(None)
        elif wl.io_dtype == "bf16":
            out.append(round_to_bf16_bits(a.astype(np.float32)).reshape(shape))
        else:
            out.append(a.astype(np.float32))
    return Inputs(wl, out[0], out[1], out[2], filt)
