"""Build the codec library ``libentropack.so`` in-tree with nvcc for sm_100a.

Usage: ``python -m dit_weight_compression_b200.build [-v]`` (``-v`` prints ptxas register and
shared-memory usage).  Every source compiles to its own object in ``_build/`` in parallel (the
decode kernels compile as one unit per output container and table layout, from decode_unit.cu),
then one link makes the shared library.  The host encoder is compiled without floating-point contraction so its
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
PLAIN = ["api.cpp", "encoder.cpp", "decode.cu", "encode_gpu.cu"]
# The decode kernels: decode_unit.cu once per output container (OutKind 0..6) and table layout.
UNIT_OUTS = range(7)
UNIT_LAYS = (10, 11, 12, 13, 14, 15)
HEADERS = ["format.h", "blob.h", "tables.h", "decode_launch.h", "decode_device.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def jobs() -> list[tuple[str, str, list[str]]]:
    """(object name, source, extra defines) of every object the library links."""
    out = [(src, src, []) for src in PLAIN]
    for o in UNIT_OUTS:
        for lay in UNIT_LAYS:
            out.append((f"decode_unit_{o}_{lay}.cu", "decode_unit.cu", [f"-DEP_UNIT_OUT={o}", f"-DEP_UNIT_LAY={lay}"]))
    return out


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _obj(name: str) -> str:
    return os.path.join(OBJ, name + ".o")


def compile_command(job: tuple[str, str, list[str]], verbose: bool = False) -> list[str]:
    name, src, defines = job
    cmd = [nvcc(), "-O3", "-std=c++17", *ARCH, "-lineinfo",
           "-Xcompiler", "-fPIC,-O2,-ffp-contract=off,-fno-fast-math", *defines,
           "-I", os.path.join(ROOT, "include"), "-I", CSRC, "-c", os.path.join(CSRC, src), "-o", _obj(name)]
    if verbose and src.endswith(".cu"):
        cmd += ["-Xptxas", "-v"]
    return cmd


def link_command() -> list[str]:
    return [nvcc(), *ARCH, "-shared", "-o", LIB, *[_obj(name) for name, _, _ in jobs()], "-lpthread"]


def _deps_time() -> float:
    deps = [os.path.join(CSRC, f) for f in HEADERS] + [os.path.join(ROOT, "include", "entropack.h")]
    return max(os.path.getmtime(d) for d in deps)


def _stale_jobs(force: bool) -> list[tuple[str, str, list[str]]]:
    if force:
        return jobs()
    hdr = _deps_time()
    out = []
    for job in jobs():
        o = _obj(job[0])
        if not os.path.exists(o) or os.path.getmtime(o) < max(hdr, os.path.getmtime(os.path.join(CSRC, job[1]))):
            out.append(job)
    return out


def stale() -> bool:
    if not os.path.exists(LIB) or _stale_jobs(False):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(_obj(name)) > t for name, _, _ in jobs())


def build(verbose: bool = False, force: bool = False) -> str:
    todo = _stale_jobs(force)
    if todo or not os.path.exists(LIB) or stale():
        os.makedirs(OBJ, exist_ok=True)
        # the largest units first, so the tail of the parallel build is short
        todo.sort(key=lambda j: (j[1] != "decode_unit.cu", "_4_" in j[0], "_14." in j[0] or "_13." in j[0]))
        workers = max(1, min(len(todo), os.cpu_count() or 1))

        def run(job):
            r = subprocess.run(compile_command(job, verbose), capture_output=True, text=True)
            return job[0], r

        failed = []
        with ThreadPoolExecutor(workers) as pool:
            for name, r in pool.map(run, todo):
                if r.stdout or r.stderr:
                    sys.stderr.write(r.stdout + r.stderr)
                if r.returncode != 0:
                    failed.append(name)
        if failed:
            raise RuntimeError(f"nvcc failed on {', '.join(failed)}")
        subprocess.run(link_command(), check=True)
    return LIB


if __name__ == "__main__":
    build(verbose="-v" in sys.argv, force=True)
    print(LIB)
