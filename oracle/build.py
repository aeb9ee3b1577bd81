"""Builds the CPU oracle shared library (test infrastructure only).

Plain g++, no fast-math and no floating-point contraction, so that every
product and sum is the IEEE float64 operation written in the source.
"""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "lmoe_oracle.cpp")
LIB_PATH = os.path.join(HERE, "liblmoe_oracle.so")


def build_oracle(force: bool = False) -> str:
    if (not force and os.path.exists(LIB_PATH)
            and os.path.getmtime(LIB_PATH) >= os.path.getmtime(SRC)):
        return LIB_PATH
    cmd = ["g++", "-std=c++17", "-O2", "-fPIC", "-shared", "-pthread",
           "-ffp-contract=off", "-fno-fast-math", SRC, "-o", LIB_PATH + ".tmp"]
    subprocess.run(cmd, check=True)
    os.replace(LIB_PATH + ".tmp", LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build_oracle(force=True))
