"""Oracle of the lattice-rANS weight codec -- TEST INFRASTRUCTURE ONLY.

A ctypes binding over ``oracle.c``: a plain, slow, single-threaded C99 implementation in double
precision of the encoder, the blob format and the decoder.  Only the test suite, the smoke check
and the CPU-baseline leg of the benchmark may import this package; the product package never
does, and the two share no code.

Dtype codes follow the blob header: 1 = BF16, 2 = FP16, 3 = FP8 E4M3, 4 = FP32, 5 = INT8.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

BF16, FP16, E4M3, F32, INT8 = 1, 2, 3, 4, 5
ITEMSIZE = {BF16: 2, FP16: 2, E4M3: 1, F32: 4, INT8: 1}
NPTYPE = {BF16: np.uint16, FP16: np.uint16, E4M3: np.uint8, F32: np.uint32, INT8: np.uint8}


def build() -> str:
    """Compile oracle.c into liboracle.so (plain gcc, no fast-math, no FMA contraction)."""
    cmd = ["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-Wall", "-fPIC",
           "-shared", "-o", _LIB, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
            build()
        L = ctypes.CDLL(_LIB)
        P, I64, U64, D, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64, ctypes.c_double, ctypes.c_int
        sig = {
            "orc_compress": (I, [P, I, I64, I64, D, I64, D, ctypes.POINTER(P), ctypes.POINTER(U64)]),
            "orc_compress_ex": (I, [P, I, I64, I64, D, I64, D, I, I, ctypes.POINTER(P), ctypes.POINTER(U64)]),
            "orc_decompress_rowscaled_tiles": (I, [P, U64, I64, I64, P, P]),
            "orc_row_gain": (ctypes.c_float, [ctypes.c_float, ctypes.c_uint32]),
            "orc_row_sigma": (ctypes.c_float, [ctypes.c_float, ctypes.c_uint32]),
            "orc_decompress": (I, [P, U64, I, P]),
            "orc_decompress_tiles": (I, [P, U64, I64, I64, I, P]),
            "orc_decode_fields": (I, [P, U64, I64, I64, P]),
            "orc_actual_bpp": (D, [P, U64]),
            "orc_blob_info": (I, [P, U64, P, ctypes.POINTER(D)]),
            "orc_free": (None, [P]),
            "orc_e8_nearest_n": (None, [P, I64, P, P]),
            "orc_point_to_fields_n": (None, [P, P, I64, P]),
            "orc_fields_to_point_n": (None, [P, P, I64, P]),
            "orc_dtype_to_f64_n": (None, [P, I, I64, P]),
            "orc_round_f32_n": (None, [P, I64, P]),
            "orc_cvt_f32_array": (None, [P, U64, I, P]),
            "orc_quantize_table": (None, [P, P, I]),
            "orc_build_tables16": (None, [P, P, I]),
            "orc_encode_tile": (U64, [P, P, I64, P, I, P, U64]),
            "orc_decode_tile": (I, [P, U64, I64, P, I, P, P, P]),
            "orc_estimate_bpp": (D, [P, I, I64, I64, D, I64, I, I]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _buf(b: bytes):
    return ctypes.cast(ctypes.c_char_p(b), ctypes.c_void_p)


# ---- codec -------------------------------------------------------------------------------------

def compress(bits: np.ndarray, dtype: int, target_bpp: float, steps_per_tile: int = 0,
             scale: float = 0.0, rd_refine: bool = False, prob_bits: int = 0) -> bytes:
    """Encode a 2-D array of dtype bit patterns; returns the blob bytes.  rd_refine turns on the
    per-row rate-distortion refinement (off by default); prob_bits is the frequency total's
    width, 12 (the default, also selected by 0) or 10."""
    bits = np.ascontiguousarray(bits)
    assert bits.ndim == 2 and bits.dtype == NPTYPE[dtype]
    out = ctypes.c_void_p()
    n = ctypes.c_uint64()
    rc = lib().orc_compress_ex(_ptr(bits), dtype, bits.shape[0], bits.shape[1], float(target_bpp),
                               int(steps_per_tile), float(scale), int(bool(rd_refine)), int(prob_bits),
                               ctypes.byref(out), ctypes.byref(n))
    if rc != 0:
        raise ValueError(f"oracle compress failed: {rc}")
    data = ctypes.string_at(out, n.value)
    lib().orc_free(out)
    return data


def blob_info(blob: bytes) -> dict:
    info = np.zeros(8, np.int64)
    s = ctypes.c_double()
    rc = lib().orc_blob_info(_buf(blob), len(blob), _ptr(info), ctypes.byref(s))
    if rc != 0:
        raise ValueError(f"oracle: bad blob ({rc})")
    rows, cols, S, ntiles, dtype, pb, off_offsets, off_stream = (int(v) for v in info)
    return dict(rows=rows, cols=cols, S=S, n_tiles=ntiles, dtype=dtype, prob_bits=pb, scale=s.value,
                off_offsets=off_offsets, off_stream=off_stream, V=rows * ((cols + 7) // 8))


def decompress(blob: bytes, dtype_out: int | None = None) -> np.ndarray:
    """Decode the whole blob; returns a rows x cols array of dtype_out bit patterns."""
    info = blob_info(blob)
    dtype_out = dtype_out or info["dtype"]
    out = np.zeros((info["rows"], info["cols"]), NPTYPE[dtype_out])
    rc = lib().orc_decompress(_buf(blob), len(blob), dtype_out, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle decompress failed: {rc}")
    return out


def decompress_tiles(blob: bytes, t0: int, t1: int, dtype_out: int, out: np.ndarray) -> None:
    """Decode tiles [t0, t1) into out (full-size rows x cols array); other elements untouched."""
    assert out.flags.c_contiguous and out.dtype == NPTYPE[dtype_out]
    rc = lib().orc_decompress_tiles(_buf(blob), len(blob), t0, t1, dtype_out, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle decompress_tiles failed: {rc}")


def decompress_rowscaled(blob: bytes, t0: int = 0, t1: int = -1, out: np.ndarray | None = None):
    """The FP8 container with a per-row scale: (E4M3 payload bits, rows x cols uint8; sigma, rows
    float32).  Tiles [t0, t1) are decoded into `out` (a new zero array when None)."""
    info = blob_info(blob)
    if out is None:
        out = np.zeros((info["rows"], info["cols"]), np.uint8)
    assert out.flags.c_contiguous and out.dtype == np.uint8 and out.shape == (info["rows"], info["cols"])
    sigma = np.zeros(info["rows"], np.float32)
    rc = lib().orc_decompress_rowscaled_tiles(_buf(blob), len(blob), t0, t1, _ptr(out), _ptr(sigma))
    if rc != 0:
        raise ValueError(f"oracle decompress_rowscaled failed: {rc}")
    return out, sigma


def row_gain(alpha: float, m2: int) -> float:
    """Per-row factor of the FP8 row-scaled payload: RNE_fp32(896 / m2) with alpha's sign."""
    return lib().orc_row_gain(float(alpha), int(m2))


def row_sigma(alpha: float, m2: int) -> float:
    """Per-row scale of the FP8 row-scaled payload: RNE_fp32(|alpha| m2 / 896)."""
    return lib().orc_row_sigma(float(alpha), int(m2))


def decode_fields(blob: bytes, t0: int = 0, t1: int = -1) -> np.ndarray:
    """(V, 9) int16: column 0 the coset bit, columns 1..8 the fields f1..f8."""
    info = blob_info(blob)
    out = np.zeros((info["V"], 9), np.int16)
    rc = lib().orc_decode_fields(_buf(blob), len(blob), t0, t1, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle decode_fields failed: {rc}")
    return out


def actual_bpp(blob: bytes) -> float:
    return lib().orc_actual_bpp(_buf(blob), len(blob))


def estimate_bpp(bits: np.ndarray, dtype: int, scale: float, steps_per_tile: int,
                 full_sample: bool, prob_bits: int = 0) -> float:
    bits = np.ascontiguousarray(bits)
    return lib().orc_estimate_bpp(_ptr(bits), dtype, bits.shape[0], bits.shape[1], float(scale),
                                  int(steps_per_tile), int(full_sample), int(prob_bits))


# ---- components --------------------------------------------------------------------------------

def e8_nearest(t: np.ndarray):
    t = np.ascontiguousarray(t, np.float64).reshape(-1, 8)
    y = np.zeros_like(t)
    c = np.zeros(len(t), np.int32)
    lib().orc_e8_nearest_n(_ptr(t), len(t), _ptr(y), _ptr(c))
    return y, c


def point_to_fields(y: np.ndarray, coset: np.ndarray) -> np.ndarray:
    y = np.ascontiguousarray(y, np.float64).reshape(-1, 8)
    c = np.ascontiguousarray(coset, np.int32)
    f = np.zeros((len(y), 8), np.int32)
    lib().orc_point_to_fields_n(_ptr(y), _ptr(c), len(y), _ptr(f))
    return f


def fields_to_point(coset: np.ndarray, f: np.ndarray) -> np.ndarray:
    c = np.ascontiguousarray(coset, np.int32)
    f = np.ascontiguousarray(f, np.int32).reshape(-1, 8)
    y = np.zeros((len(f), 8), np.float64)
    lib().orc_fields_to_point_n(_ptr(c), _ptr(f), len(f), _ptr(y))
    return y


def dtype_to_f64(bits: np.ndarray, dtype: int) -> np.ndarray:
    bits = np.ascontiguousarray(bits, NPTYPE[dtype])
    out = np.zeros(bits.shape, np.float64)
    lib().orc_dtype_to_f64_n(_ptr(bits), dtype, bits.size, _ptr(out))
    return out


def round_f32(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, np.float64)
    out = np.zeros(v.shape, np.uint32)
    lib().orc_round_f32_n(_ptr(v), v.size, _ptr(out))
    return out


def cvt_f32(bits: np.ndarray, dtype_out: int) -> np.ndarray:
    bits = np.ascontiguousarray(bits, np.uint32)
    out = np.zeros(bits.shape, NPTYPE[dtype_out])
    lib().orc_cvt_f32_array(_ptr(bits), bits.size, dtype_out, _ptr(out))
    return out


def quantize_table(counts: np.ndarray, prob_bits: int = 12) -> np.ndarray:
    counts = np.ascontiguousarray(counts, np.uint64)
    assert counts.shape == (256,)
    q = np.zeros(256, np.uint16)
    lib().orc_quantize_table(_ptr(counts), _ptr(q), int(prob_bits))
    return q


def build_tables16(counts: np.ndarray, prob_bits: int = 12) -> np.ndarray:
    """The 16 context tables (16 x 256) from symbol counts (16 x 256): contexts 0 and 8 quantised
    together as the joint (coset, f1) table, the others one by one; totals 2^prob_bits."""
    counts = np.ascontiguousarray(counts, np.uint64).reshape(16, 256)
    q = np.zeros((16, 256), np.uint16)
    lib().orc_build_tables16(_ptr(counts), _ptr(q), int(prob_bits))
    return q


def encode_tile(sym9: np.ndarray, raw8: np.ndarray, q16: np.ndarray, prob_bits: int = 12) -> bytes:
    sym9 = np.ascontiguousarray(sym9, np.uint8).reshape(-1, 9)
    raw8 = np.ascontiguousarray(raw8, np.int16).reshape(-1, 8)
    q16 = np.ascontiguousarray(q16, np.uint16).reshape(16, 256)
    n = lib().orc_encode_tile(_ptr(sym9), _ptr(raw8), len(sym9), _ptr(q16), int(prob_bits), None, 0)
    if n == 0:
        raise ValueError("oracle encode_tile failed")
    out = np.zeros(n, np.uint8)
    lib().orc_encode_tile(_ptr(sym9), _ptr(raw8), len(sym9), _ptr(q16), int(prob_bits), _ptr(out), n)
    return out.tobytes()


def decode_tile(tile: bytes, nvec: int, q16: np.ndarray, prob_bits: int = 12):
    """Returns (rc, sym9, raw8, final_states); raw8 is meaningful only where sym9 is the escape."""
    q16 = np.ascontiguousarray(q16, np.uint16).reshape(16, 256)
    sym9 = np.zeros((nvec, 9), np.uint8)
    raw8 = np.zeros((nvec, 8), np.int16)
    st = np.zeros(32, np.uint32)
    rc = lib().orc_decode_tile(_buf(tile), len(tile), nvec, _ptr(q16), int(prob_bits), _ptr(sym9), _ptr(raw8),
                               _ptr(st))
    return rc, sym9, raw8, st
