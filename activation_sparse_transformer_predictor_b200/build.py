"""Build libspark.so (the C-ABI library) in-tree with nvcc for sm_100a, and
libspark_debug.so, the same sources compiled with SPARK_DEBUG (bounds-checked
kernels, see spark_debug_violations in include/spark.h).

Usage: ``python -m activation_sparse_transformer_predictor_b200.build [--verbose]``.
The libraries are written next to this file so that they travel with the source tree.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libspark.so")
DEBUG_LIB = os.path.join(PKG, "libspark_debug.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def _command(out: str, debug: bool, verbose: bool) -> list[str]:
    cmd = [NVCC, *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), "-I", CSRC, "-shared", "-o", out, *sources()]
    if debug:
        cmd.insert(1, "-DSPARK_DEBUG")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def build(force: bool = False, verbose: bool = False, debug: bool = True) -> str:
    """Compile the release library (and, with ``debug``, the bounds-checked one)
    where a source is newer than it; both nvcc runs go side by side.  Returns
    the release library's path."""
    targets = [(LIB, False)] + ([(DEBUG_LIB, True)] if debug else [])
    procs = []
    for lib, dbg in targets:
        if not force and not _stale(lib):
            continue
        tmp = lib + f".tmp{os.getpid()}"
        cmd = _command(tmp, dbg, verbose)
        if verbose:
            print(" ".join(cmd))
        procs.append((subprocess.Popen(cmd), tmp, lib, cmd))
    failed = None
    for proc, tmp, lib, cmd in procs:
        if proc.wait() != 0:
            failed = failed or subprocess.CalledProcessError(proc.returncode, cmd)
        else:
            os.replace(tmp, lib)
    if failed is not None:
        raise failed
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
    print(DEBUG_LIB)
