"""Build the sm_100a CUDA library libsqint8.so in this package directory.

One translation unit (csrc/sqint8.cu) holds every kernel and the C ABI of
include/sqint8.h.  Compiled with nvcc for sm_100a only, without fast math,
with the CUDA runtime linked statically; the driver's tensor-map encoder is
looked up at run time, so no libcuda link is needed.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "sqint8.cu")
LIB = os.path.join(HERE, "libsqint8.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-shared", "-Xptxas", "-v", "--expt-relaxed-constexpr",
         "-I", os.path.join(ROOT, "include")]


def sources():
    c = os.path.join(HERE, "csrc")
    return [os.path.join(c, f) for f in os.listdir(c)] + [os.path.join(ROOT, "include", "sqint8.h")]


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and os.path.exists(LIB) and all(
            os.path.getmtime(LIB) >= os.path.getmtime(s) for s in sources()):
        return LIB
    cmd = [NVCC, *FLAGS, SRC, "-o", LIB + ".tmp"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building libsqint8.so")
    if verbose:
        sys.stderr.write(r.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
