"""Build libhyena_nd.so (sm_100a) in-tree with nvcc.

    python -m dimensional_long_convolution_b200.build [--force] [--bounds]

Each translation unit under csrc/ is compiled in parallel, then linked into
dimensional_long_convolution_b200/libhyena_nd.so.  The build is skipped when
the library is newer than every source.

--bounds builds the index-checked variant instead, libhyena_nd_bounds.so
beside it: the same sources with HYENA_ND_BOUNDS defined and relocatable
device code (one table of the call's buffers shared by every unit), in which
every kernel access to a caller buffer or to shared memory is checked and a
violation is reported as HYENA_ND_ERR_DEVICE_BOUNDS instead of touching
memory (csrc/hnd_bounds.cuh).  It is for tests, not for speed.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import time
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libhyena_nd.so")
BUILD_BOUNDS = os.path.join(ROOT, "_build_bounds")
LIB_BOUNDS = os.path.join(PKG, "libhyena_nd_bounds.so")
BOUNDS_FLAGS = ["-DHYENA_ND_BOUNDS", "-rdc=true"]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
              "--expt-relaxed-constexpr", "-Xptxas", "-warn-spills"]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found")
    return path


def sources() -> list:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps() -> list:
    pats = ["*.cu", "*.cuh", "*.h", "*.inc", "*.py"]
    out = []
    for p in pats:
        out += glob.glob(os.path.join(CSRC, p))
    out += glob.glob(os.path.join(INCLUDE, "*.h"))
    out.append(os.path.abspath(__file__))
    return out


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(d) <= t for d in _deps())


def build(force: bool = False, extra_flags=None, verbose: bool = False, jobs: int = 0, bounds: bool = False) -> str:
    lib = LIB_BOUNDS if bounds else LIB
    bdir = BUILD_BOUNDS if bounds else BUILD
    if not force and up_to_date(lib):
        return lib
    t0 = time.time()
    subprocess.check_call([sys.executable, os.path.join(CSRC, "gen_tables.py"), os.path.join(CSRC, "hnd_twiddles.inc")])
    os.makedirs(bdir, exist_ok=True)
    flags = NVCC_FLAGS + list(extra_flags or []) + (BOUNDS_FLAGS if bounds else [])
    exe = nvcc()

    def compile_one(src: str) -> str:
        obj = os.path.join(bdir, os.path.basename(src) + ".o")
        cmd = [exe] + ARCH + flags + ["-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError("nvcc failed for %s:\n%s\n%s" % (src, " ".join(cmd), res.stderr))
        if verbose and res.stderr.strip():
            print(res.stderr)
        return obj

    srcs = sources()
    with cf.ThreadPoolExecutor(max_workers=jobs or min(len(srcs), os.cpu_count() or 4)) as ex:
        objs = list(ex.map(compile_one, srcs))
    tmp = lib + ".tmp"
    cmd = [exe] + ARCH + (["-rdc=true"] if bounds else []) + ["-shared", "-o", tmp] + objs + ["-lcudart"]
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    # stamp the library with the build's start, so that a source edited while
    # it compiled leaves it out of date
    os.utime(lib, (t0, t0))
    return lib


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--bounds", action="store_true", help="build the index-checked variant libhyena_nd_bounds.so")
    args = ap.parse_args()
    print(build(force=args.force, verbose=args.verbose, bounds=args.bounds))


if __name__ == "__main__":
    main()
