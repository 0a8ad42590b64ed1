#!/usr/bin/env python
"""Throughput of the gated nD FFT long convolution on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config I] [--impl ours|reference]

One step = one call of hyena_nd_fftconv_batched over the whole batch of the
workload (gate-in, padded forward nD FFT, spectral product, inverse nD FFT,
crop and output gate for every (b, c) volume).  The per-channel spectrum is
produced once beforehand by hyena_nd_filter_spectrum (the filter call is not
part of the metric).  Inputs are seeded synthetic tensors of the benchmark
grid; three input sets (q, k, v, y and spectrum) rotate between steps so no
step finds its data in L2.

Metric: voxel*channels per second (B*C*prod(n) per step), GB/s of the
unavoidable HBM bytes (q, k, v, y once each plus the spectrum once) and the
fraction of the measured B200 copy bandwidth.  With N > 1 (torchrun), every
rank runs the same workload on its own GPU (independent volumes, no
collective): weak scaling, value = all ranks' voxel*channels / max time.

--impl reference times the float64 CPU oracle (test infrastructure) on a
bounded sample of the same workload: the slow reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from dimensional_long_convolution_b200 import workloads as W  # noqa: E402
from dimensional_long_convolution_b200.parallel import max_over_ranks, shard_range  # noqa: E402

METRIC = "gated nD FFT long-conv voxel*channels/s"
UNIT = "voxel*ch/s"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0      # B200 HBM3e nominal (DGX figure); the measured copy bandwidth is the roofline peak
REPEATS = 5                   # the timed steps run as this many equal segments; their median is reported beside the total


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=0, help="timed steps (0 = enough for about 3 s)")
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", type=lambda x: int(x) if x.isdigit() else x, default=2,
                    help="benchmark grid index (0..4) or workload name")
    ap.add_argument("--also", default="0,1,3,4,seq1d_1m_b1_c64_bf16", help="extra grids measured kernel-only, comma separated "
                    "(suite indices or workload names, e.g. seq1d_1m_b1_c64_bf16)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--sets", type=int, default=3, help="rotating input sets")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    return ap.parse_args()


def unavoidable_bytes(wl) -> int:
    elt = 2 if wl.io_dtype == "bf16" else 4
    P = [2 * n for n in wl.dims]
    half = int(np.prod(P[:-1])) * (P[-1] // 2 + 1)
    return 4 * wl.B * wl.C * wl.voxels * elt + wl.C * half * 8


def plan_summary(setup) -> dict:
    """Tier, waves and launches of the measured problem, from the library's
    host-side plan (no device work)."""
    info = setup.H.plan_info(setup.op.p)
    return {k: info[k] for k in ("tier", "wave", "waves", "launches", "split")}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "dimensional_long_convolution_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh", ".h", ".inc")) and name != "hnd_twiddles.inc":
            with open(os.path.join(csrc, name), "rb") as fh:
                h.update(name.encode() + fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload_name: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
        e = d.get(workload_name)
        if e and e.get("source_sha") == kernel_source_sha():
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


def recorded_pipes(workload_name: str):
    """FP32-pipe and issue fractions of a step (time-weighted over its
    kernels) from a committed ncu summary taken on the current kernel
    sources, else None."""
    path = os.path.join(ROOT, "profiles", "pipes.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
        e = d.get(workload_name)
        if e and e.get("source_sha") == kernel_source_sha():
            return {k: e[k] for k in ("fma_pipe_frac", "issue_frac", "dram_bytes_per_step") if k in e}
    except Exception:
        pass
    return None


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, smax, power, reasons = [], [], [], set()
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[2]))
                smax.append(float(f[3]))
                power.append(float(f[4]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        # "under load": samples drawing more than the idle floor
        pw = np.array(power)
        load = np.array(sm)[pw >= max(pw.min() + 0.25 * (pw.max() - pw.min()), 0)]
        return {"sm_mhz": float(np.median(load if load.size else sm)), "sm_max_mhz": float(max(smax)),
                "reasons": sorted(reasons), "samples": len(sm), "power_w_max": float(pw.max())}


# ------------------------------------------------------------------ CPU side
def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_pair_fn(wl, inp):
    """Time the float64 oracle on one (b, c) volume per call (O2 route)."""
    from oracle import hyena_nd_oracle as O
    chans = [0]
    K = O.implicit_kernel(inp.filt, wl.dims, channels=chans)
    S = O.spectrum_full(K, wl.dims)
    q = inp.as_f64("q")[:1, :1]
    k = inp.as_f64("k")[:1, :1]
    v = inp.as_f64("v")[:1, :1]

    def one():
        O.conv_dft(q, k, v, S, wl.dims)
    return one


def cpu_baseline(wl, inp, seconds: float):
    one = oracle_pair_fn(wl, inp)
    one()                                   # warm (DFT matrices, BLAS threads)
    t0 = time.perf_counter()
    n = 0
    while True:
        one()
        n += 1
        dt = time.perf_counter() - t0
        if dt >= seconds or n >= wl.B * wl.C:
            break
    return {"value": n * wl.voxels / dt, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
            "sample": "%d of %d (b,c) volumes of %s through the float64 padded-DFT oracle, %.1f s" %
                      (n, wl.B * wl.C, wl.name, dt)}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    wl = W.workload(args.config)
    inp = W.make_inputs(wl)
    one = oracle_pair_fn(wl, inp)
    for _ in range(max(args.warmup, 0)):
        one()
    K = args.steps if args.steps > 0 else 5
    t0 = time.perf_counter()
    for _ in range(K):
        one()
    dt = time.perf_counter() - t0
    value = K * wl.voxels / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": 1e3 * dt / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "dims": list(wl.dims), "B": wl.B, "C": wl.C, "io_dtype": wl.io_dtype,
                   "step": "one (b,c) volume of the workload per step"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                         "sample": "one (b,c) volume of %s per step, %d steps" % (wl.name, K)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# ------------------------------------------------------------------ GPU side
class Setup:
    def __init__(self, wl, nsets, device):
        import torch
        from dimensional_long_convolution_b200 import hyena_nd as H
        self.wl = wl
        self.torch = torch
        self.H = H
        self.op = H.HyenaND(wl.dims, wl.B, wl.C, wl.io_dtype, device=device)
        base = W.make_inputs(wl)
        self.inp0 = base
        f = base.filt
        self.op.set_filter(*(torch.from_numpy(a) for a in (f.W1, f.b1, f.W2, f.b2, f.alpha)), f.decay_scale,
                           f.num_freqs)
        self.sets = []
        for s in range(nsets):
            inp = base if s == 0 else W.make_inputs(wl, seed=wl.seed + 1000 * s)
            t = [self._dev(getattr(inp, n), device) for n in ("q", "k", "v")]
            y = torch.empty_like(t[0])
            spec = self.op.spectrum if s == 0 else self.op.spectrum.clone()
            self.sets.append((t[0], t[1], t[2], y, spec))
        torch.cuda.synchronize(device)
        self.launches = self.step(0)

    def _dev(self, a, device):
        torch = self.torch
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
        return torch.from_numpy(a).to(device)

    def step(self, i):
        q, k, v, y, spec = self.sets[i % len(self.sets)]
        self.op(q, k, v, y=y, spectrum=spec)
        return self.H.last_launch_count()


def time_steps(setup, K, stream, segments: int = 1):
    """Device time of K back-to-back steps (CUDA events on the launching
    stream).  With segments > 1 the same K steps are split into that many
    consecutive equal parts with an event between parts; returns the total
    and the per-step time of each part."""
    torch = setup.torch
    segments = max(1, min(segments, K))
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(segments + 1)]
    bounds = [K * j // segments for j in range(segments + 1)]
    ev[0].record(stream)
    for j in range(segments):
        for i in range(bounds[j], bounds[j + 1]):
            setup.step(i)
        ev[j + 1].record(stream)
    ev[-1].synchronize()
    parts = [ev[j].elapsed_time(ev[j + 1]) / max(1, bounds[j + 1] - bounds[j]) for j in range(segments)]
    if segments == 1:
        return ev[0].elapsed_time(ev[-1])
    return ev[0].elapsed_time(ev[-1]), parts


def time_filter_call(setup, device, stream, n: int) -> float:
    """ms per call 1 (filter spectrum) with device-resident weights: the MLP
    on the offset grid, the window, the padded transform and the packing.
    The spectrum it rewrites is the same one (same weights)."""
    torch = setup.torch
    f = setup.inp0.filt
    wdev = [torch.from_numpy(a).to(device) for a in (f.W1, f.b1, f.W2, f.b2, f.alpha)]
    setup.op.set_filter(*wdev, f.decay_scale, f.num_freqs)
    fa, fb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    fa.record(stream)
    for _ in range(n):
        setup.op.set_filter(*wdev, f.decay_scale, f.num_freqs)
    fb.record(stream)
    fb.synchronize()
    return fa.elapsed_time(fb) / n


def run_ours(args):
    import torch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    wl = W.workload(args.config)
    setup = Setup(wl, args.sets, device)
    stream = torch.cuda.current_stream(device)

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(device)

    # warm-up, then size K for about 3 s of timed work unless given
    for i in range(max(args.warmup, 3)):
        setup.step(i)
    torch.cuda.synchronize(device)
    probe = time_steps(setup, 20, stream) / 20.0
    K = args.steps if args.steps > 0 else int(max(50, min(200000, 3000.0 / max(probe, 1e-3))))
    if dist is not None:
        kt = torch.tensor([K], device=device)
        dist.all_reduce(kt, op=dist.ReduceOp.MAX)
        K = int(kt.item())

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier()
    ms, parts = time_steps(setup, K, stream, REPEATS)
    barrier()
    clocks.stop()
    ms_max = max_over_ranks(ms, dist, device)
    # weak scaling: the global batch is world x B samples, rank r owns its slice
    shard = shard_range(world * wl.B, rank, world)

    units = wl.B * wl.C * wl.voxels
    value = world * units * K / (ms_max / 1e3)
    peak, peak_kind = measured_peaks()
    ub = unavoidable_bytes(wl)
    step_ms = ms / K
    achieved = ub / (step_ms / 1e3) / 1e9
    launches = setup.launches

    # end to end: pinned host buffers, H2D of q, k, v and D2H of y inside the
    # timed region, every step.  Steps are pipelined the way a streaming
    # caller would run them: two device buffer sets; the inputs of step i + 1
    # go up (copy stream) while step i computes and the output of step i - 1
    # comes down (a second copy stream, the other PCIe direction).
    q0, k0, v0, y0, spec0 = setup.sets[0]
    hq, hk, hv = (x.cpu().pin_memory() for x in (q0, k0, v0))
    hy = [torch.empty(y0.shape, dtype=y0.dtype).pin_memory() for _ in range(2)]
    dbuf = [(q0, k0, v0, y0), tuple(torch.empty_like(x) for x in (q0, k0, v0, y0))]
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    E = max(3, min(K, 30))

    def e2e_step(i):
        j = i % 2
        dq, dk, dv, dy = dbuf[j]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_comp[j])          # step i - 2 has consumed these inputs
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            ev_in[j].record(s_in)
        stream.wait_event(ev_in[j])
        if i >= 2:
            stream.wait_event(ev_out[j])             # step i - 2's output has left this buffer
        setup.op(dq, dk, dv, y=dy, spectrum=spec0)
        ev_comp[j].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[j])
            hy[j].copy_(dy, non_blocking=True)
            ev_out[j].record(s_out)

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize(device)
    barrier()
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ea.record(s_in)
    for i in range(E):
        e2e_step(i)
    eb.record(s_out)
    eb.synchronize()
    torch.cuda.synchronize(device)
    barrier()
    te = max_over_ranks(ea.elapsed_time(eb), dist, device)
    elt = 2 if wl.io_dtype == "bf16" else 4
    e2e = {"value": world * units * E / (te / 1e3), "unit": UNIT,
           "h2d_bytes_per_step": 3 * units * elt, "d2h_bytes_per_step": units * elt,
           "ms_per_step": te / E,
           "pipelining": "two device buffer sets; step i + 1's H2D overlaps step i's kernels and step i - 1's D2H"}

    # warm: the same grid with one input set reused every step, so whatever of
    # q, k, v, y and the spectrum L2 keeps between steps is found there
    warm = None
    if args.sets > 1:
        q1, k1, v1, y1, s1 = setup.sets[0]
        saved = setup.sets
        setup.sets = [(q1, k1, v1, y1, s1)]
        for i in range(3):
            setup.step(i)
        Kw = max(REPEATS, min(K, 2000))
        tw, wparts = time_steps(setup, Kw, stream, REPEATS)
        setup.sets = saved
        wparts.sort()
        warm = {"ms_per_step": tw / Kw, "median_ms_per_step": wparts[len(wparts) // 2], "steps": Kw,
                "note": "one input set reused every step (L2 may keep part of it)"}

    also = []
    for tok in [x for x in args.also.split(",") if x.strip() != ""]:
        j = int(tok) if tok.strip().isdigit() else tok.strip()
        if j == args.config:
            continue
        wj = W.workload(j)
        sj = Setup(wj, args.sets, device)
        for i in range(5):
            sj.step(i)
        torch.cuda.synchronize(device)
        pj = time_steps(sj, 10, stream) / 10.0
        Kj = int(max(20, min(20000, 1500.0 / max(pj, 1e-3))))
        msj, pparts = time_steps(sj, Kj, stream, REPEATS)
        sm = msj / Kj
        pparts.sort()
        ubj = unavoidable_bytes(wj)
        entry = {"workload": wj.name, "value": wj.B * wj.C * wj.voxels / (sm / 1e3), "unit": UNIT,
                 "ms_per_step": sm, "median_ms_per_step": pparts[len(pparts) // 2],
                 "gbs": ubj / (sm / 1e3) / 1e9, "hbm_frac": ubj / (sm / 1e3) / 1e9 / peak,
                 "hbm_frac_nominal": ubj / (sm / 1e3) / 1e9 / NOMINAL_HBM_GBS,
                 "launches_per_step": sj.launches, "steps": Kj, "plan": plan_summary(sj)}
        pj_rec = recorded_pipes(wj.name)
        if pj_rec:
            entry["profile"] = pj_rec
        entry["filter_call_ms"] = time_filter_call(sj, device, stream, 3)
        entry["filter_call_conv_steps"] = entry["filter_call_ms"] / sm
        also.append(entry)
        del sj
        torch.cuda.empty_cache()

    call1_ms = time_filter_call(setup, device, stream, 5)
    filter_call = {"ms_per_call": call1_ms, "conv_steps_per_call": call1_ms / (ms / K),
                   "note": "not in the metric: the spectrum is computed once per filter update"}

    # backward (dq, dk, dv for a loss gradient dy) on the same grid, timed
    # apart from the metric; algorithmic bytes: q, k, v, dy read, dq, dk, dv
    # written, the spectrum read twice (the dq and the adjoint convolutions)
    dy0 = torch.empty_like(y0).copy_(setup.sets[-1][0])
    for _ in range(3):
        setup.op.backward(q0, k0, v0, dy0, spectrum=spec0)
    bwd_launches = setup.H.last_launch_count()
    ba, bb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    NB = max(5, min(200, K // 3))
    ba.record(stream)
    for _ in range(NB):
        setup.op.backward(q0, k0, v0, dy0, spectrum=spec0)
    bb.record(stream)
    bb.synchronize()
    bwd_ms = ba.elapsed_time(bb) / NB
    for _ in range(2):
        setup.op.kernel_grad(q0, k0, v0, dy0)
    ka, kb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    NKG = 5
    ka.record(stream)
    for _ in range(NKG):
        setup.op.kernel_grad(q0, k0, v0, dy0)
    kb.record(stream)
    kb.synchronize()
    kgrad_ms = ka.elapsed_time(kb) / NKG
    bwd_bytes = 7 * units * elt + 2 * (ub - 4 * units * elt)
    backward = {"ms_per_step": bwd_ms, "value": units / (bwd_ms / 1e3), "unit": UNIT,
                "launches_per_step": bwd_launches, "gbs": bwd_bytes / (bwd_ms / 1e3) / 1e9,
                "hbm_frac": bwd_bytes / (bwd_ms / 1e3) / 1e9 / peak,
                "note": "two convolutions: dq, then the adjoint writing dk and dv",
                "kernel_grad_ms": kgrad_ms}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, setup.inp0, args.cpu_seconds)

    kernel_desc = {1: "fused single-CTA kernel", 3: "three multi-pass kernels per wave"}
    parts.sort()
    pipes = recorded_pipes(wl.name)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_max / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": wl.io_dtype + " io, f32 compute", "data": "synthetic",
        "config": {"workload": wl.name, "dims": list(wl.dims), "B": wl.B, "C": wl.C, "io_dtype": wl.io_dtype,
                   "parallelism": "batch-sharded x%d (rank 0 samples %d..%d of %d; independent volumes, no "
                                  "collective)" % (world, shard[0], shard[1] - 1, world * wl.B),
                   "l2": "%d rotating input sets of %.0f MB each (> 126 MB L2 between reuses)" %
                         (args.sets, ub / 1e6),
                   "plan": plan_summary(setup)},
        "gbs": ub * K / (ms_max / 1e3) / 1e9 * world,
        "median_ms_per_step": parts[len(parts) // 2],
        "repeats_ms_per_step": parts,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "frac_nominal": achieved / NOMINAL_HBM_GBS, "nominal_peak": NOMINAL_HBM_GBS,
                     "traffic": recorded_traffic(wl.name), "peak_kind": peak_kind,
                     "fp32_pipe_frac": pipes.get("fma_pipe_frac") if pipes else None,
                     "issue_frac": pipes.get("issue_frac") if pipes else None,
                     "kernel": "step (%d launch%s per step: %s)" % (
                         launches, "" if launches == 1 else "es", kernel_desc.get(launches, "multi-pass waves")),
                     "algorithmic_bytes_per_step": ub, "kernel_source_sha": kernel_source_sha()},
        "gpu_launches": int(launches * K),
        "clocks": clocks.summary(),
        "e2e": e2e,
        "warm": warm,
        "filter_call": filter_call,
        "backward": backward,
        "also": also,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line))
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
