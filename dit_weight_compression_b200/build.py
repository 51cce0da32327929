"""Build the codec library ``libentropack.so`` in-tree with nvcc for sm_100a.

Usage: ``python -m dit_weight_compression_b200.build [-v]`` (``-v`` prints ptxas register and
shared-memory usage).  Every source compiles to its own object in ``_build/`` in parallel (the
decode kernel's output containers are separate translation units), then one link makes the
shared library.  The host encoder is compiled without floating-point contraction so its
arithmetic is plain IEEE double precision.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OBJ = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libentropack.so")
SOURCES = ["api.cpp", "encoder.cpp", "decode.cu", "decode_bf16.cu", "decode_fp16.cu", "decode_e4m3.cu",
           "decode_f32.cu", "decode_i8.cu", "decode_fields.cu", "decode_e4m3row.cu", "encode_gpu.cu"]
HEADERS = ["format.h", "blob.h", "tables.h", "decode_launch.h", "decode_device.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _obj(src: str) -> str:
    return os.path.join(OBJ, src + ".o")


def compile_command(src: str, verbose: bool = False) -> list[str]:
    cmd = [nvcc(), "-O3", "-std=c++17", *ARCH, "-lineinfo",
           "-Xcompiler", "-fPIC,-O2,-ffp-contract=off,-fno-fast-math",
           "-I", os.path.join(ROOT, "include"), "-I", CSRC, "-c", os.path.join(CSRC, src), "-o", _obj(src)]
    if verbose and src.endswith(".cu"):
        cmd += ["-Xptxas", "-v"]
    return cmd


def link_command() -> list[str]:
    return [nvcc(), *ARCH, "-shared", "-o", LIB, *[_obj(s) for s in SOURCES], "-lpthread"]


def _deps_time() -> float:
    deps = [os.path.join(CSRC, f) for f in HEADERS] + [os.path.join(ROOT, "include", "entropack.h")]
    return max(os.path.getmtime(d) for d in deps)


def _stale_objects(force: bool) -> list[str]:
    if force:
        return list(SOURCES)
    hdr = _deps_time()
    out = []
    for s in SOURCES:
        o = _obj(s)
        if not os.path.exists(o) or os.path.getmtime(o) < max(hdr, os.path.getmtime(os.path.join(CSRC, s))):
            out.append(s)
    return out


def stale() -> bool:
    if not os.path.exists(LIB) or _stale_objects(False):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(_obj(s)) > t for s in SOURCES)


def build(verbose: bool = False, force: bool = False) -> str:
    todo = _stale_objects(force)
    if todo or not os.path.exists(LIB) or stale():
        os.makedirs(OBJ, exist_ok=True)
        jobs = max(1, min(len(todo), os.cpu_count() or 1))

        def run(src):
            r = subprocess.run(compile_command(src, verbose), capture_output=True, text=True)
            return src, r

        failed = []
        with ThreadPoolExecutor(jobs) as pool:
            for src, r in pool.map(run, todo):
                if r.stdout or r.stderr:
                    sys.stderr.write(r.stdout + r.stderr)
                if r.returncode != 0:
                    failed.append(src)
        if failed:
            raise RuntimeError(f"nvcc failed on {', '.join(failed)}")
        subprocess.run(link_command(), check=True)
    return LIB


if __name__ == "__main__":
    build(verbose="-v" in sys.argv, force=True)
    print(LIB)
