"""Builds liblmoe.so (the C-ABI CUDA library) in-tree for sm_100a.

    python -m mixture_experts_layer_64_b200.build [--ptxas-verbose]
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB_PATH = os.path.join(HERE, "liblmoe.so")
SOURCES = [os.path.join(CSRC, "lmoe.cu"), os.path.join(CSRC, "noalloc.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")] + [
    os.path.join(ROOT, "include", "lmoe.h")]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def build_library(force: bool = False, verbose: bool = False) -> str:
    if (not force and os.path.exists(LIB_PATH)
            and os.path.getmtime(LIB_PATH) >= max(os.path.getmtime(p) for p in DEPS)):
        return LIB_PATH
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr",
           "-I", os.path.join(ROOT, "include"), "-o", LIB_PATH + ".tmp", *SOURCES]
    if verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    subprocess.run(cmd, check=True)
    os.replace(LIB_PATH + ".tmp", LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build_library(force=True, verbose="--ptxas-verbose" in sys.argv))
