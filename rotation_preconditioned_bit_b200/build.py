"""Build libharp.so in-tree with nvcc for sm_100a (no GPU needed)."""

from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libharp.so")
SOURCES = [os.path.join(CSRC, f) for f in ("harp_kernels.cu", "harp_api.cpp", "harp_static_ws.cu")]
HEADERS = [os.path.join(CSRC, "harp_internal.h"), os.path.join(INCLUDE, "harp.h")]
CUDA_HOME = os.environ.get("CUDA_HOME", "/usr/local/cuda")
NVCC = os.path.join(CUDA_HOME, "bin", "nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2,-Wall",
    "-Xptxas", "-warn-spills",
    "-shared", "-cudart", "shared",
    "-Xlinker", f"-rpath,{CUDA_HOME}/lib64",
    "-I", INCLUDE, "-I", CSRC,
]


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in SOURCES + HEADERS)


def build(force: bool = False, verbose: bool = False) -> str:
    if force or stale():
        cmd = [NVCC, *FLAGS, "-o", LIB, *SOURCES]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.check_call(cmd)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    print(LIB)
