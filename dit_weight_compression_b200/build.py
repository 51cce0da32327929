"""Build the codec library ``libentropack.so`` in-tree with nvcc for sm_100a.

Usage: ``python -m dit_weight_compression_b200.build [-v]`` (``-v`` prints ptxas register and
shared-memory usage).  The host encoder is compiled without floating-point contraction so its
arithmetic is plain IEEE double precision.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libentropack.so")
SOURCES = ["api.cpp", "encoder.cpp", "decode.cu", "encode_gpu.cu"]
HEADERS = ["format.h", "blob.h", "tables.h"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(verbose: bool = False) -> list[str]:
    cmd = [nvcc(), "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
           "-Xcompiler", "-fPIC,-O2,-ffp-contract=off,-fno-fast-math", "-shared",
           "-I", os.path.join(ROOT, "include"), "-I", CSRC, "-o", LIB]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    cmd += ["-lpthread"]
    return cmd


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(ROOT, "include", "entropack.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(verbose: bool = False, force: bool = False) -> str:
    if force or stale():
        subprocess.run(command(verbose), check=True)
    return LIB


if __name__ == "__main__":
    build(verbose="-v" in sys.argv, force=True)
    print(LIB)
