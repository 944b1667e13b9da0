"""Build libqg.so in-tree: nvcc for sm_100a (CUDA sources) + the host packer, one shared object.

Usage: python -m quant_dequant_gemv_q4_b200.build [--force]
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libqg.so")
SOURCES = [os.path.join(CSRC, "qg_api.cu"), os.path.join(CSRC, "qg_pack.cpp")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC)) if f.endswith((".cuh", ".h"))] \
    + [os.path.join(INCLUDE, "qg.h")]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_cmd(out: str, extra=()) -> list[str]:
    return [NVCC, *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-shared",
            "-I", INCLUDE, *extra, "-o", out, *SOURCES]


def build(force: bool = False, verbose: bool = False) -> str:
    stale = force or not os.path.exists(LIB) or any(
        os.path.getmtime(d) > os.path.getmtime(LIB) for d in DEPS)
    if stale:
        tmp = LIB + f".tmp{os.getpid()}"
        extra = ["-Xptxas", "-v"] if verbose else []
        subprocess.check_call(nvcc_cmd(tmp, extra))
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
