"""Build libmxmoe.so in-tree with nvcc for sm_100a.

The library is one CUDA translation unit (csrc/mxmoe.cu) with a C ABI
(include/mxmoe.h); cudart is linked statically so the .so only needs the
NVIDIA driver at run time.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libmxmoe.so")
SOURCES = [os.path.join(HERE, "csrc", f)
           for f in ("mxmoe.cu", "mx_common.cuh", "quant.cuh", "gemm.cuh", "sm100.cuh", "route.cuh")]
HEADER = os.path.join(ROOT, "include", "mxmoe.h")


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in SOURCES + [HEADER])


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not needs_build():
        return LIB
    cmd = [
        nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
        "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include"),
        "-o", LIB + ".tmp", os.path.join(HERE, "csrc", "mxmoe.cu"), "-lcudart_static", "-ldl", "-lrt", "-lpthread",
    ]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
