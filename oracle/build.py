"""Build the CPU oracle shared library (test infrastructure only).

Compiles sq_oracle.cpp with strict IEEE settings: no fast math and no
floating-point contraction, so every float operation rounds once as written.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "sq_oracle.cpp")
LIB = os.path.join(HERE, "libsqoracle.so")

FLAGS = ["-O3", "-march=x86-64-v3", "-std=c++17", "-ffp-contract=off",
         "-fno-fast-math", "-fPIC", "-shared", "-pthread"]


def build(force: bool = False) -> str:
    deps = [SRC, os.path.join(HERE, "sq_oracle.h")]
    if not force and os.path.exists(LIB) and all(
            os.path.getmtime(LIB) >= os.path.getmtime(d) for d in deps):
        return LIB
    cmd = ["g++", *FLAGS, SRC, "-o", LIB + ".tmp"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
