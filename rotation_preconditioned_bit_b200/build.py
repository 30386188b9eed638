"""Build libharp.so in-tree with nvcc for sm_100a (no GPU needed).

Each source compiles to its own object in parallel (the kernels dominate the
build time), then nvcc links the shared library. Objects go to a scratch
folder next to the library and are not part of the package.
"""

from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libharp.so")
OBJDIR = os.path.join(HERE, "_build")
SOURCES = [os.path.join(CSRC, f) for f in ("harp_kernels.cu", "harp_pass.cu", "harp_api.cpp", "harp_static_ws.cu",
                                              "harp_theta.cu", "harp_short.cu", "harp_rows.cu")]
HEADERS = [os.path.join(CSRC, "harp_internal.h"), os.path.join(CSRC, "harp_quant_dev.cuh"),
           os.path.join(CSRC, "harp_tc.cuh"),
           os.path.join(INCLUDE, "harp.h")]
CUDA_HOME = os.environ.get("CUDA_HOME", "/usr/local/cuda")
NVCC = os.path.join(CUDA_HOME, "bin", "nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ARCH + [
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2,-Wall",
    "-Xptxas", "-warn-spills",
    "-I", INCLUDE, "-I", CSRC,
]
LDFLAGS = ARCH + ["-shared", "-cudart", "shared", "-Xlinker", f"-rpath,{CUDA_HOME}/lib64"]


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in SOURCES + HEADERS)


def _obj(src: str) -> str:
    return os.path.join(OBJDIR, os.path.basename(src) + ".o")


def build(force: bool = False, verbose: bool = False) -> str:
    if force or stale():
        os.makedirs(OBJDIR, exist_ok=True)
        cmds = [[NVCC, *CFLAGS, "-c", s, "-o", _obj(s)] for s in SOURCES]
        if verbose:
            for c in cmds:
                print(" ".join(c), file=sys.stderr)
        with ThreadPoolExecutor(max_workers=len(cmds)) as ex:
            codes = list(ex.map(subprocess.call, cmds))
        if any(codes):
            raise subprocess.CalledProcessError(max(codes), cmds[codes.index(max(codes))])
        link = [NVCC, *LDFLAGS, "-o", LIB, *[_obj(s) for s in SOURCES]]
        if verbose:
            print(" ".join(link), file=sys.stderr)
        subprocess.check_call(link)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    print(LIB)
