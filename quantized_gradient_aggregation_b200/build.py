"""Build libqga.so (sm_100a) in-tree with nvcc.

    python quantized_gradient_aggregation_b200/build.py [--force] [--verbose]

(Run it by path: importing the package loads the library this script builds.)

The library is plain CUDA C++ behind the C ABI of include/qga.h; no torch
headers are involved.  ``-fmad=false`` keeps every floating-point expression
free of contraction (the kernels also spell their additions, subtractions,
multiplications and divisions with the round-to-nearest intrinsics).
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libqga.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-fmad=false",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
    "-shared",
]


def nvcc() -> str:
    home = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    path = os.path.join(home, "bin", "nvcc")
    return path if os.path.exists(path) else "nvcc"


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + [os.path.join(INCLUDE, "qga.h")]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every source to an object in parallel (one nvcc per file,
    under _build/), then link the shared library."""
    if not force and up_to_date():
        return LIB
    objdir = os.path.join(PKG, "_build")
    os.makedirs(objdir, exist_ok=True)
    compile_flags = [f for f in NVCC_FLAGS if f != "-shared"]
    jobs = []
    for src in sources():
        obj = os.path.join(objdir, os.path.splitext(os.path.basename(src))[0] + f".{os.getpid()}.o")
        cmd = [nvcc(), *compile_flags, "-I", INCLUDE, "-c", "-o", obj, src]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        jobs.append((obj, subprocess.Popen(cmd)))
    failed = [obj for obj, p in jobs if p.wait() != 0]
    objs = [obj for obj, _ in jobs]
    try:
        if failed:
            raise subprocess.CalledProcessError(1, f"nvcc ({len(failed)} of {len(jobs)} sources failed)")
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.run([nvcc(), *NVCC_FLAGS, "-o", tmp, *objs], check=True)
        os.replace(tmp, LIB)
    finally:
        for obj in objs:
            if os.path.exists(obj):
                os.remove(obj)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="--verbose" in sys.argv)
    print(LIB)
