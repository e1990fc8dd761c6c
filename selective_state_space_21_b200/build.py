"""Build libmambascan.so in-tree with nvcc for sm_100a.

    python -m selective_state_space_21_b200.build [--force] [--verbose-ptxas]
"""
from __future__ import annotations

import argparse
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIBDIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIBDIR, "libmambascan.so")
MICRO_SRC = os.path.join(CSRC, "micro", "throughput.cu")
MICRO_LIB = os.path.join(LIBDIR, "libmambamicro.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
    "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-cudart", "static",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def deps():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + [
        os.path.join(ROOT, "include", "mamba_scan.h")]


#: The files that define the staged forward and backward kernels and their
#: launches (plus the compiler flags): a stored profile of those kernels stays
#: valid while these are unchanged.
STAGED_KERNEL_FILES = ("fwd_staged.cuh", "bwd_staged.cuh", "common.cuh", "tma.cuh", "tcgen05.cuh")


def source_digest(files=None) -> str:
    """Short hash of the sources the library is built from -- all of them, or
    only ``files`` (names under csrc/) -- and of the nvcc flags (used to tell
    whether a stored profile still describes the current kernels)."""
    import hashlib
    h = hashlib.sha256()
    h.update(" ".join(NVCC_FLAGS).encode())
    paths = deps() if files is None else [os.path.join(CSRC, f) for f in files]
    for p in paths:
        h.update(os.path.basename(p).encode())
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in deps())


def build_micro(force: bool = False) -> str:
    """Build libmambamicro.so, the instruction-throughput microbenchmark that
    ``bench.py --micro`` runs (not part of the scan library)."""
    if not force and os.path.exists(MICRO_LIB) and \
            os.path.getmtime(MICRO_LIB) >= os.path.getmtime(MICRO_SRC):
        return MICRO_LIB
    os.makedirs(LIBDIR, exist_ok=True)
    tmp = MICRO_LIB + f".tmp{os.getpid()}"
    subprocess.check_call([NVCC, *NVCC_FLAGS, MICRO_SRC, "-o", tmp])
    os.replace(tmp, MICRO_LIB)
    return MICRO_LIB


DEBUG_LIB = os.path.join(LIBDIR, "libmambascan_debug.so")


def build_debug(force: bool = False) -> str:
    """Build libmambascan_debug.so: the same library with MAMBA_DEBUG_BOUNDS,
    whose kernels check their computed indices against the buffers and record
    a wrong one in the sticky status (MAMBA_ERR_OUT_OF_BOUNDS) instead of
    making the access."""
    if not force and os.path.exists(DEBUG_LIB) and \
            all(os.path.getmtime(p) <= os.path.getmtime(DEBUG_LIB) for p in deps()):
        return DEBUG_LIB
    os.makedirs(LIBDIR, exist_ok=True)
    tmp = DEBUG_LIB + f".tmp{os.getpid()}"
    subprocess.check_call([NVCC, *NVCC_FLAGS, "-DMAMBA_DEBUG_BOUNDS", "-I",
                           os.path.join(ROOT, "include"), *sources(), "-o", tmp])
    os.replace(tmp, DEBUG_LIB)
    return DEBUG_LIB


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    build_micro(force)
    if not force and not stale():
        return LIB
    os.makedirs(LIBDIR, exist_ok=True)
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC, *NVCC_FLAGS, "-I", os.path.join(ROOT, "include")]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    cmd += [*sources(), "-o", tmp]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--debug-bounds", action="store_true",
                    help="also build the bounds-checking libmambascan_debug.so")
    args = ap.parse_args()
    print(build(force=args.force, verbose_ptxas=args.verbose_ptxas))
    if args.debug_bounds:
        print(build_debug(force=args.force))
    sys.exit(0)
