"""Builds libeta.so (the CUDA kernels + C ABI) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libeta.so")
SOURCES = [os.path.join(CSRC, "eta.cu")]
DEPS = SOURCES + sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")) + \
    [os.path.join(ROOT, "include", "eta.h")]


def nvcc_cmd(out: str, extra=()) -> list:
    nvcc = os.environ.get("NVCC", "nvcc")
    return [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
            "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC,-fvisibility=hidden", "-shared",
            "-I", os.path.join(ROOT, "include"), "-I", CSRC, "-o", out, *SOURCES, *extra]


def build(force: bool = False, verbose: bool = False) -> str:
    stale = force or not os.path.exists(LIB) or any(os.path.getmtime(d) > os.path.getmtime(LIB) for d in DEPS)
    if stale:
        tmp = LIB + ".tmp.%d" % os.getpid()
        cmd = nvcc_cmd(tmp, ["-Xptxas", "-v"] if verbose else [])
        subprocess.check_call(cmd)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
