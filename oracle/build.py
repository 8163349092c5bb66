"""Build the CPU oracle shared library (oracle/liboracle.so) with g++.

Test infrastructure: the oracle is only ever loaded by the test suite, the
smoke check and the benchmark's CPU-baseline / reference arm.

The library is compiled with -O2 and -ffp-contract=off so that every multiply
and add is rounded exactly as written, with std::thread workers so that callers can
spread independent output rows (forward) or images (backward) over host cores.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "dcn4_ref.cpp")
HDR = os.path.join(HERE, "dcn4_ref.h")
LIB = os.path.join(HERE, "liboracle.so")


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    lib_t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > lib_t for f in (SRC, HDR, __file__))


def build(force: bool = False) -> str:
    """Compile liboracle.so if it is missing or older than its sources."""
    if force or needs_build():
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [
            os.environ.get("CXX", "g++"), "-std=c++17", "-O2", "-ffp-contract=off",
            "-pthread", "-fPIC", "-shared", "-Wall", "-Wextra", "-o", tmp, SRC,
        ]
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
