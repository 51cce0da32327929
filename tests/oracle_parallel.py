"""Tile-parallel oracle decodes for the full-size parity tests.

Every tile decodes on its own ("EntroPack lattice compression", section "Encoding and
reconstruction"), so the oracle can decode a large blob in tile ranges on several host cores and
the pieces are the oracle's whole-blob decode.  One pool of worker processes serves the whole test
session; it is started with `spawn`, so the workers inherit no CUDA state from a test process that
has used the GPU.  A blob reaches the workers through a temporary file.  Each worker decodes its
tile range into a lazily zero-filled full-size array (untouched pages cost no memory) and returns
only the element range those tiles cover, which is contiguous when the column count is a
multiple of 8.
"""
from __future__ import annotations

import atexit
import multiprocessing as mp
import os
import tempfile

import numpy as np

import oracle

_POOL = None
_WORKERS = 0
_CACHE = {}   # in a worker: path -> blob bytes of the file last read there


def _blob(path: str) -> bytes:
    b = _CACHE.get(path)
    if b is None:
        _CACHE.clear()
        with open(path, "rb") as fh:
            b = fh.read()
        _CACHE[path] = b
    return b


def _work(job):
    path, kind, t0, t1, dtype = job
    blob = _blob(path)
    info = oracle.blob_info(blob)
    per = 32 * info["S"]
    v0, v1 = t0 * per, min(t1 * per, info["V"])
    if kind == "fields":
        f = oracle.decode_fields(blob, t0, t1)
        return v0, f[v0:v1].copy()
    if kind == "rowscaled":
        out, sigma = oracle.decompress_rowscaled(blob, t0, t1)
        return v0, out.reshape(-1)[8 * v0:8 * v1].copy(), sigma
    out = np.zeros((info["rows"], info["cols"]), oracle.NPTYPE[dtype])
    oracle.decompress_tiles(blob, t0, t1, dtype, out)
    return v0, out.reshape(-1)[8 * v0:8 * v1].copy()


def _cores() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return os.cpu_count() or 1


def _pool():
    global _POOL, _WORKERS
    if _POOL is None:
        oracle.lib()                                  # build the oracle once, before the workers load it
        _WORKERS = max(1, min(_cores(), 32))
        _POOL = mp.get_context("spawn").Pool(_WORKERS)
        atexit.register(_POOL.terminate)
    return _POOL


def decode(blob: bytes, kind: str = "values", dtype: int | None = None):
    """The oracle's decode of the whole blob, computed tile-parallel.
    kind = "values": rows x cols array of dtype bit patterns (default: the blob's dtype);
           "fields": (V, 9) int16 fields; "rowscaled": (E4M3 payload bits, per-row sigma)."""
    info = oracle.blob_info(blob)
    assert info["cols"] % 8 == 0, "tile ranges map to contiguous elements only without column padding"
    dtype = dtype or info["dtype"]
    pool = _pool()
    n = info["n_tiles"]
    k = max(1, min(_WORKERS, n))
    bounds = [n * i // k for i in range(k + 1)]
    fd, path = tempfile.mkstemp(suffix=".blob")
    try:
        with os.fdopen(fd, "wb") as fh:
            fh.write(blob)
        jobs = [(path, kind, bounds[i], bounds[i + 1], dtype) for i in range(k) if bounds[i] < bounds[i + 1]]
        parts = pool.map(_work, jobs)
    finally:
        os.unlink(path)
    if kind == "fields":
        out = np.zeros((info["V"], 9), np.int16)
        for v0, f in parts:
            out[v0:v0 + len(f)] = f
        return out
    flat = np.zeros(info["rows"] * info["cols"], np.uint8 if kind == "rowscaled" else oracle.NPTYPE[dtype])
    for part in parts:
        flat[8 * part[0]:8 * part[0] + len(part[1])] = part[1]
    out = flat.reshape(info["rows"], info["cols"])
    if kind == "rowscaled":
        return out, parts[0][2]
    return out
