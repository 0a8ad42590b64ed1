"""Host-only checks of the C ABI: the library loads, exports every symbol that
include/hyena_nd.h declares, reports sizes, and rejects bad arguments before
touching the GPU (no call here reaches a kernel launch)."""
import os
import re

import numpy as np
import pytest

from dimensional_long_convolution_b200 import hyena_nd as H
from dimensional_long_convolution_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "hyena_nd.h")).read()
    return sorted(set(re.findall(r"HYENA_ND_API\s+[\w\s\*]+?\b(hyena_nd_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = H.load()
    names = _declared()
    assert len(names) == len(H.EXPORTED) == 18
    assert set(names) == set(H.EXPORTED)
    for n in names:
        assert getattr(lib, n) is not None


def test_status_strings():
    assert H.status_string(0) == "HYENA_ND_OK"
    assert H.status_string(6) == "HYENA_ND_ERR_DEVICE_TIMEOUT"
    assert H.status_string(99) == "HYENA_ND_ERR_UNKNOWN"


@pytest.mark.parametrize("i", range(5))
def test_sizes_of_the_benchmark_grids(i):
    wl = W.workload(i)
    p = H.problem(wl.dims, wl.B, wl.C, H.BF16 if wl.io_dtype == "bf16" else H.F32)
    P = [2 * n for n in wl.dims]
    half = 1
    for a in P[:-1]:
        half *= a
    half *= P[-1] // 2 + 1
    assert H.spectrum_bytes(p) == wl.C * half * 8
    ws = H.workspace_bytes(p)
    assert ws >= 256 and ws % 16 == 0
    assert H.workspace_bytes(p) == ws          # pure function of the descriptor


@pytest.mark.parametrize("dims,B,C,dt,circ,want", [
    ((64, 64), 1, 1, 0, 0, True),
    ((300, 300), 1, 1, 0, 0, False),          # not a power of two
    ((512, 8), 1, 1, 0, 0, False),            # a 2D axis above 256
    ((512,), 1, 1, 0, 0, True),               # long 1D context
    ((131072,), 2, 4, 1, 1, True),            # longest two-level split, circular
    ((1 << 26,), 1, 1, 0, 0, True),           # longest 1D grid (three levels)
    ((1 << 27,), 1, 1, 0, 0, False),          # above the long 1D limit
    ((3000,), 1, 1, 0, 0, False),             # long 1D, not a power of two
    ((4, 8), 1, 1, 0, 0, False),              # below 8
    ((256, 64, 64), 1, 1, 0, 0, False),       # outer 3D axis above 128
    ((64, 64), 0, 1, 0, 0, False),            # B < 1
    ((64, 64), 1, 1, 7, 0, False),            # unknown dtype
    ((64, 64), 1, 1, 0, 1, True),             # circular mode
])
def test_workspace_bytes_is_zero_for_invalid_problems(dims, B, C, dt, circ, want):
    p = H.problem(dims, B, C, dt, circ)
    assert (H.workspace_bytes(p) > 0) == want
    assert (H.spectrum_bytes(p) > 0) == want


def test_rank_zero_and_four_are_invalid():
    p = H.problem((64, 64), 1, 1)
    p.ndim = 0
    assert H.workspace_bytes(p) == 0
    p.ndim = 4
    assert H.workspace_bytes(p) == 0


# fake, never dereferenced device addresses (argument checks run first)
A = 0x7F0000000000
STEP = 1 << 30


def _ptrs():
    return [A + i * STEP for i in range(6)]


def _call(p, q, k, v, s, y, ws, wsb, sbs=0):
    return H.fftconv_batched(p, q, k, v, s, sbs, y, ws, wsb, 0)


def test_invalid_arguments_are_rejected_before_launch():
    p = H.problem((64, 64), 2, 3)
    q, k, v, s, y, ws = _ptrs()
    wsb = H.workspace_bytes_for(p, H.CALL_CONV)
    assert _call(p, 0, k, v, s, y, ws, wsb) == H.ERR_INVALID_ARG
    assert _call(p, q, k, v, 0, y, ws, wsb) == H.ERR_INVALID_ARG
    assert _call(p, q, k, v, s, y, 0, wsb) == H.ERR_INVALID_ARG
    assert _call(p, q + 4, k, v, s, y, ws, wsb) == H.ERR_MISALIGNED
    assert _call(p, q, k, v, s, y + 8, ws, wsb) == H.ERR_MISALIGNED
    assert _call(p, q, k, v, s, y, ws, wsb - 16) == H.ERR_WORKSPACE_TOO_SMALL
    assert _call(p, q, k, v, s, q, ws, wsb) == H.ERR_INVALID_ARG          # y aliases q
    assert _call(p, q, k, v, s, k + 64, ws, wsb) == H.ERR_INVALID_ARG     # y overlaps k
    assert _call(p, q, k, v, s, y, ws, wsb, sbs=-16) == H.ERR_INVALID_ARG
    assert _call(p, q, k, v, s, y, ws, wsb, sbs=8) == H.ERR_MISALIGNED
    bad = H.problem((48, 64), 2, 3)
    assert _call(bad, q, k, v, s, y, ws, wsb) == H.ERR_UNSUPPORTED
    circ = H.problem((64, 64), 2, 3, circular=2)
    assert _call(circ, q, k, v, s, y, ws, wsb) == H.ERR_INVALID_ARG


def test_backward_arguments_are_rejected_before_launch():
    p = H.problem((64, 64), 2, 3)
    q, k, v, s, dy, ws = _ptrs()
    dq, dk, dv = (A + i * STEP for i in (6, 7, 8))
    wsb = H.workspace_bytes_for(p, H.CALL_CONV)

    def bwd(*args, sbs=0, wsb_=wsb, prob=p):
        a = dict(q=q, k=k, v=v, s=s, dy=dy, dq=dq, dk=dk, dv=dv, ws=ws)
        a.update(args[0] if args else {})
        return H.fftconv_backward(prob, a["q"], a["k"], a["v"], a["s"], sbs, a["dy"], a["dq"], a["dk"], a["dv"],
                                  a["ws"], wsb_, 0)

    assert bwd({"dy": 0}) == H.ERR_INVALID_ARG
    assert bwd({"dv": 0}) == H.ERR_INVALID_ARG
    assert bwd({"dq": dq + 8}) == H.ERR_MISALIGNED
    assert bwd({"dk": q}) == H.ERR_INVALID_ARG            # output aliases an input
    assert bwd({"dv": dy + 64}) == H.ERR_INVALID_ARG      # output overlaps dy
    assert bwd({"dk": dq}) == H.ERR_INVALID_ARG           # two outputs alias
    assert bwd(wsb_=wsb - 16) == H.ERR_WORKSPACE_TOO_SMALL
    assert bwd(sbs=-16) == H.ERR_INVALID_ARG
    assert bwd(sbs=8) == H.ERR_MISALIGNED
    assert bwd(prob=H.problem((48, 64), 2, 3)) == H.ERR_UNSUPPORTED


def test_kernel_grad_arguments_are_rejected_before_launch():
    p = H.problem((32, 16), 2, 3)
    q, k, v, dy, dK, ws = _ptrs()
    wsb = H.workspace_bytes(p)
    assert H.kernel_grad(p, q, k, v, 0, dK, ws, wsb) == H.ERR_INVALID_ARG
    assert H.kernel_grad(p, q, k, v, dy, 0, ws, wsb) == H.ERR_INVALID_ARG
    assert H.kernel_grad(p, q, k, v, dy, dK + 4, ws, wsb) == H.ERR_MISALIGNED
    assert H.kernel_grad(p, q, k, v, dy, dK, ws, wsb - 16) == H.ERR_WORKSPACE_TOO_SMALL
    assert H.kernel_grad(p, q, k, v, dy, k + 64, ws, wsb) == H.ERR_INVALID_ARG     # dK overlaps k
    assert H.kernel_grad(H.problem((24, 16), 2, 3), q, k, v, dy, dK, ws, wsb) == H.ERR_UNSUPPORTED


def test_workspace_covers_the_kernel_gradient():
    """The workspace of every grid holds at least one channel's kernel-gradient
    grids: B padded complex grids and one accumulator."""
    for i in range(5):
        wl = W.workload(i)
        p = H.problem(wl.dims, wl.B, wl.C, H.BF16 if wl.io_dtype == "bf16" else H.F32)
        P = int(np.prod([2 * n for n in wl.dims]))
        assert H.workspace_bytes(p) >= (wl.B + 1) * P * 8


def _long_1d_split(n):
    """Factors of 2n: two levels up to 2^18, else three, each at most 2^9,
    the larger shares first."""
    lg = (2 * n).bit_length() - 1
    m = 2 if lg <= 18 else 3
    out, left = [], lg
    for a in range(m):
        share = -(-left // (m - a))
        out.append(1 << share)
        left -= share
    return out


@pytest.mark.parametrize("n,B,C", [(512, 2, 3), (4096, 1, 8), (131072, 2, 100), (1 << 23, 1, 2), (1 << 26, 1, 1)])
def test_long_1d_sizes(n, B, C):
    """Long 1D spectra are stored per channel pair: (A, D) = ((K_a + K_b)/2,
    (K_a - K_b)/2) as two complex64 values for the pencils kap = 0 .. Po/2 of
    the split (Po = P / Pc, Pc the last factor), i.e. about half of the 2n
    frequencies; the workspace holds at least one pair's padded grid (one
    wave) and the kernel-gradient grids of one channel; the natural export
    stays n + 1."""
    p = H.problem((n,), B, C, H.F32)
    sp = _long_1d_split(n)
    assert int(np.prod(sp)) == 2 * n and max(sp) <= 512
    Pc, Po = sp[-1], 2 * n // sp[-1]
    assert H.spectrum_bytes(p) == (C + 1) // 2 * (Po // 2 + 1) * Pc * 16
    assert H.spectrum_bytes(p) == (C + 1) // 2 * (2 * n * 8 + 16 * Pc)   # half the frequencies, two values each
    ws = H.workspace_bytes(p)
    assert ws >= 256 + max(2 * n * 8, (B + 1) * 2 * n * 8)
    # the largest of: a 48 MiB conv wave, 256 MiB of kernel-gradient grids,
    # 2.25 GiB of filter grids (each at least one volume or channel), plus tables
    assert ws <= 256 + max(48 << 20, 256 << 20, 2304 << 20, (B + 1) * 2 * n * 8, 2 * n * 8) + (1 << 20)


def test_long_1d_spectrum_conversion_uses_the_natural_size():
    """The natural half spectrum of a long 1D grid and the library's pair
    layout differ in size; the overlap check measures each buffer by its own
    size."""
    n, C = 1024, 2
    p = H.problem((n,), 1, C)
    nat = C * (n + 1) * 8
    nat16 = (nat + 15) // 16 * 16
    assert H.spectrum_bytes(p) == (64 // 2 + 1) * 32 * 16     # 2048 = 64 x 32, one channel pair
    assert H.spectrum_import(p, A, A + nat16 - 16, 0) == H.ERR_INVALID_ARG
    assert H.spectrum_export(p, A + nat16 - 16, A, 0) == H.ERR_INVALID_ARG


def test_static_scratch_call_limits_long_1d():
    """The no-allocation call runs long 1D grids while one volume's split grid
    (16 bytes per token) fits its 16 MiB array: 2^21 tokens do not, and 2^27
    is beyond every tier.  Both are refused on the host (fake pointers)."""
    q, k, v, s, y, ws = _ptrs()
    assert H.fftconv_batched_static(H.problem((1 << 21,), 1, 1), q, k, v, s, 0, y, 0) == \
        H.ERR_WORKSPACE_TOO_SMALL
    assert H.fftconv_batched_static(H.problem((1 << 27,), 1, 1), q, k, v, s, 0, y, 0) == H.ERR_UNSUPPORTED


@pytest.mark.parametrize("i", range(5))
def test_workspace_stays_within_the_chunk_budgets(i):
    """Every benchmark grid's workspace is the largest of its scratch parts:
    a conv wave (64 MiB), a filter chunk (2.25 GiB plus first-layer tables) and
    a kernel-gradient chunk (256 MiB), each at least one volume or channel."""
    wl = W.workload(i)
    p = H.problem(wl.dims, wl.B, wl.C, H.BF16 if wl.io_dtype == "bf16" else H.F32)
    P = int(np.prod([2 * n for n in wl.dims]))
    one = max(8 * P * (wl.B + 1), 8 * P)
    tables = 5 * 511 * 128 * 4        # three axes' tables and the last axis' sine and cosine
    assert H.workspace_bytes(p) <= 256 + max(2304 << 20, one) + 256 + tables


@pytest.mark.parametrize("i,tier,waves,launches,streams", [
    (0, "fused_2d", 1, 1, 1), (1, "fused_2d", 1, 1, 1), (2, "multi_2d", 7, 21, 3), (3, "multi_3d", 13, 39, 3),
    (4, "multi_3d", 32, 96, 3)])
def test_plan_info_of_the_benchmark_grids(i, tier, waves, launches, streams):
    """The plan the calls run, read on the host: the launch counts are the
    ones the GPU tests and the bench observe; multi-pass grids with several
    waves run them round-robin on three streams, each wave in a third of
    64 MiB."""
    wl = W.workload(i)
    p = H.problem(wl.dims, wl.B, wl.C, H.BF16 if wl.io_dtype == "bf16" else H.F32)
    info = H.plan_info(p)
    assert (info["tier"], info["waves"], info["launches"], info["streams"]) == (tier, waves, launches, streams)
    assert info["workspace_bytes"] == H.workspace_bytes(p)
    assert info["spectrum_bytes"] == H.spectrum_bytes(p)
    if waves > 1:       # balanced waves of whole channels' samples
        assert info["wave"] * (waves - 1) < wl.B * wl.C <= info["wave"] * waves
        assert info["wave"] % wl.B == 0


@pytest.mark.parametrize("n,B,C,levels,split,waves", [
    (256, 1, 4, 0, [1, 1, 1], 1), (512, 2, 3, 2, [32, 32, 1], 1), (1 << 17, 1, 60, 2, [512, 512, 1], 4),
    (1 << 20, 1, 64, 3, [128, 128, 128], 32), (1 << 23, 1, 8, 3, [256, 256, 256], 4),
    (1 << 26, 1, 1, 3, [512, 512, 512], 1)])
def test_plan_info_of_long_1d(n, B, C, levels, split, waves):
    """Long 1D waves count channel-pair grids (8 bytes per padded point
    each).  Grids that need several waves of the 48 MiB budget, and of which
    three fit it, run in waves of a third of it on three streams: 2^17
    tokens, C = 60 -> 30 grids of 2 MiB -> 4 waves of 8; 2^20 tokens, C = 64
    -> 32 grids of 16 MiB -> 32 waves of one; 2^23 tokens (128 MiB grids) ->
    one grid per wave, one stream."""
    info = H.plan_info(H.problem((n,), B, C))
    assert info["split_levels"] == levels and info["split"] == split
    assert info["tier"] == ("long_1d" if n > 256 else "rows_1d")
    assert info["waves"] == waves
    assert info["streams"] == (3 if waves > 1 and 2 * n * 8 * 3 <= 48 << 20 else 1)
    if levels:
        assert info["launches"] == waves * (2 * levels - 1)
        assert int(np.prod(split)) == 2 * n


def test_plan_info_rejects_bad_problems():
    info = H.PlanInfo()
    lib = H.load()
    assert lib.hyena_nd_plan_info_get(None, H.ctypes.byref(info)) == H.ERR_INVALID_ARG
    assert lib.hyena_nd_plan_info_get(H.ctypes.byref(H.problem((64, 64), 1, 1)), None) == H.ERR_INVALID_ARG
    assert lib.hyena_nd_plan_info_get(H.ctypes.byref(H.problem((300,), 1, 1)), H.ctypes.byref(info)) == \
        H.ERR_UNSUPPORTED


def test_single_volume_call_needs_b_and_c_of_one():
    q, k, v, s, y, ws = _ptrs()
    p = H.problem((32, 32), 2, 1)
    assert H.fftconv(p, q, k, v, s, y, ws, 1 << 30, 0) == H.ERR_INVALID_ARG


def test_filter_arguments_are_checked():
    p = H.problem((32, 32), 1, 4)
    _, _, _, s, _, ws = _ptrs()
    wsb = H.workspace_bytes_for(p, H.CALL_FILTER)
    f = H.Filter()
    f.num_freqs, f.hidden = 8, 64
    f.W1 = f.b1 = f.W2 = f.b2 = f.alpha = A + 7 * STEP
    f.decay_scale, f.window = 32.0, 0
    f.window = 2
    assert H.filter_spectrum(p, f, s, ws, wsb) == H.ERR_UNSUPPORTED      # no such window
    f.window = 0
    f.hidden = 0
    assert H.filter_spectrum(p, f, s, ws, wsb) == H.ERR_UNSUPPORTED
    f.hidden = 64
    f.decay_scale = 0.0
    assert H.filter_spectrum(p, f, s, ws, wsb) == H.ERR_INVALID_ARG
    f.decay_scale = 32.0
    f.W2 = 0
    assert H.filter_spectrum(p, f, s, ws, wsb) == H.ERR_INVALID_ARG
    f.W2 = A + 7 * STEP + 2
    assert H.filter_spectrum(p, f, s, ws, wsb) == H.ERR_MISALIGNED
    f.W2 = A + 7 * STEP
    assert H.filter_spectrum(p, f, s, ws, wsb - 1) == H.ERR_WORKSPACE_TOO_SMALL


def test_film_filter_arguments_are_checked():
    p = H.problem((32, 32), 2, 4)
    _, _, _, s, _, ws = _ptrs()
    wsb = H.workspace_bytes_for(p, H.CALL_FILTER)
    sb = H.spectrum_bytes(p)
    f = H.Filter()
    f.num_freqs, f.hidden = 8, 64
    f.W1 = f.b1 = f.W2 = f.b2 = f.alpha = A + 7 * STEP
    f.decay_scale, f.window = 32.0, 0
    g = bt = A + 8 * STEP
    assert H.filter_spectrum_film(p, f, 0, bt, s, sb, ws, wsb) == H.ERR_INVALID_ARG          # no gamma
    assert H.filter_spectrum_film(p, f, g, 0, s, sb, ws, wsb) == H.ERR_INVALID_ARG           # no beta
    assert H.filter_spectrum_film(p, f, g + 2, bt, s, sb, ws, wsb) == H.ERR_MISALIGNED
    assert H.filter_spectrum_film(p, f, g, bt, s, sb - 16, ws, wsb) == H.ERR_INVALID_ARG     # stride below one spectrum
    assert H.filter_spectrum_film(p, f, g, bt, s, sb + 8, ws, wsb) == H.ERR_MISALIGNED
    assert H.filter_spectrum_film(p, f, g, bt, s, sb, ws, wsb - 1) == H.ERR_WORKSPACE_TOO_SMALL
    f.window = 2
    assert H.filter_spectrum_film(p, f, g, bt, s, sb, ws, wsb) == H.ERR_UNSUPPORTED


def test_spectrum_conversion_checks():
    p = H.problem((32, 32), 1, 4)
    nb = H.spectrum_bytes(p)
    assert H.spectrum_export(p, A, A + nb // 2, 0) == H.ERR_INVALID_ARG     # overlap
    assert H.spectrum_import(p, A + 4, A + STEP, 0) == H.ERR_MISALIGNED
    assert H.spectrum_import(p, 0, A + STEP, 0) == H.ERR_INVALID_ARG


def test_status_and_debug_calls_check_arguments():
    # a null workspace names the no-allocation call's status word, which needs
    # a device: without one the lookup fails as a CUDA error
    assert H.device_status(0, 0) == H.ERR_CUDA
    assert H.device_status(A + 4, 0) == H.ERR_MISALIGNED
    assert H.workspace_init(A, 16, 0) == H.ERR_WORKSPACE_TOO_SMALL
    assert H.debug_bounded_wait(A, 4096, 0, 0) == H.ERR_INVALID_ARG
    assert H.debug_bounded_wait(A, 8, 100, 0) == H.ERR_WORKSPACE_TOO_SMALL


@pytest.mark.parametrize("i", range(5))
def test_workspace_bytes_per_call(i):
    """Each call kind needs only its own scratch: the convolution calls their
    waves (nothing beyond the control area on the single-launch tiers), the
    filter and kernel-gradient calls their channel chunks; the largest of the
    three is hyena_nd_workspace_bytes."""
    wl = W.workload(i)
    p = H.problem(wl.dims, wl.B, wl.C, H.BF16 if wl.io_dtype == "bf16" else H.F32)
    conv, filt, kg = (H.workspace_bytes_for(p, c) for c in (H.CALL_CONV, H.CALL_FILTER, H.CALL_KERNEL_GRAD))
    assert H.workspace_bytes_for(p, H.CALL_ALL) == H.workspace_bytes(p) == max(conv, filt, kg)
    info = H.plan_info(p)
    if info["tier"] == "fused_2d":
        assert conv == 256
    else:
        per = 8 * wl.voxels * int(info["wave"])
        assert conv == 256 + info["streams"] * ((per + 255) // 256 * 256)
    assert H.workspace_bytes_for(p, 99) == 0


def test_calls_check_their_own_workspace_size():
    """Host-side rejects against each call's own figure (fake pointers: these
    return before any launch)."""
    q, k, v, s, y, ws = _ptrs()
    p = H.problem((256, 256), 2, 128, H.BF16)
    conv = H.workspace_bytes_for(p, H.CALL_CONV)
    assert conv < H.workspace_bytes(p)
    assert H.fftconv_batched(p, q, k, v, s, 0, y, ws, conv - 16, 0) == H.ERR_WORKSPACE_TOO_SMALL
    kg = H.workspace_bytes_for(p, H.CALL_KERNEL_GRAD)
    assert H.kernel_grad(p, q, k, v, s, y, ws, kg - 16, 0) == H.ERR_WORKSPACE_TOO_SMALL
