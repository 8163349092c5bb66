"""Build libdcn4.so in-tree with nvcc for sm_100a (B200).

    python deformable_convolution_sampling_b200/build.py [--force] [--ptxas-info]

(run as a script: importing the package itself needs the built library).

Compiles every .cu file under csrc/ into one shared library next to this file.
nvcc cross-compiles for sm_100a without a GPU.
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
LIB = os.path.join(PKG, "libdcn4.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
              "--expt-relaxed-constexpr"]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs() -> list[str]:
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + sorted(
        glob.glob(os.path.join(INCLUDE, "*.h"))) + [os.path.abspath(__file__)]


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in _inputs())


def nvcc() -> str:
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    path = os.path.join(cuda, "bin", "nvcc")
    return path if os.path.exists(path) else "nvcc"


def build(force: bool = False, ptxas_info: bool = False) -> str:
    """Compile libdcn4.so if it is missing or older than its sources; return its path."""
    if not (force or ptxas_info or needs_build()):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    objdir = os.path.join(PKG, "_build")
    os.makedirs(objdir, exist_ok=True)
    # one nvcc per translation unit, all at once, then one link
    procs, objs = [], []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + f".{os.getpid()}.o")
        cmd = [nvcc(), *ARCH_FLAGS, *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, "-c", "-o", obj, src]
        if ptxas_info:
            cmd.insert(1, "-Xptxas=-v")
        procs.append((src, subprocess.Popen(cmd)))
        objs.append(obj)
        if ptxas_info:  # one at a time, so the resource reports do not interleave
            procs[-1][1].wait()
    failed = [src for src, proc in procs if proc.wait() != 0]
    try:
        if failed:
            raise subprocess.CalledProcessError(1, f"nvcc {' '.join(os.path.basename(f) for f in failed)}")
        subprocess.run([nvcc(), *ARCH_FLAGS, "-shared", "-o", tmp, *objs], check=True)
        os.replace(tmp, LIB)
    finally:
        for obj in objs:
            if os.path.exists(obj):
                os.remove(obj)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, ptxas_info="--ptxas-info" in sys.argv))
