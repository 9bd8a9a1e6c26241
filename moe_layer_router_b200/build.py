"""Build libmoe_b200.so (sm_100a) in-tree with nvcc.

    python moe_layer_router_b200/build.py [--force] [--ptxas-v]
    (run by path: importing the package itself needs the built library)

The library is one translation unit (csrc/moe_api.cu) that includes the kernels.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmoe_b200.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC,-O3",
    "--expt-relaxed-constexpr",
    "-shared",
]


def sources():
    out = [os.path.join(INCLUDE, "moe.h")]
    for n in sorted(os.listdir(CSRC)):
        if n.endswith((".cu", ".cuh")):
            out.append(os.path.join(CSRC, n))
    return out


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.isabs(c) and os.path.exists(c) or not os.path.isabs(c)):
            return c
    return "nvcc"


def build(force: bool = False, verbose: bool = False, extra=None) -> str:
    srcs = sources()
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= max(os.path.getmtime(s) for s in srcs):
        return LIB
    cmd = [nvcc()] + NVCC_FLAGS + (extra or []) + [os.path.join(CSRC, "moe_api.cu"), "-o", LIB + ".tmp"]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None)
