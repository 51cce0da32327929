"""Inputs of the golden digests: small seeded matrices and the settings they are compressed with.

Only seeded input generation lives here (no codec arithmetic); both make_golden.py, which writes
the digests with the oracle, and tests/test_golden.py, which checks the library against them,
draw their inputs from this module.
"""
from __future__ import annotations

import numpy as np

import workloads as W

# name -> (what the case covers, frequency-total bits, target bpp, output containers checked)
CASES = {
    "small_bf16_pb12": ("256x256 BF16 N(0, 0.02^2) at 3.5 bpp, 12-bit totals (the usage example's shape and rate)",
                        12, 3.5, (W.BF16, W.FP16, W.E4M3, W.F32)),
    "small_bf16_pb10": ("the same with 10-bit totals", 10, 3.5, (W.BF16,)),
    "ragged_bf16": ("37x203 BF16 at 3.5 bpp: columns padded to whole vectors, a partial last tile",
                    12, 3.5, (W.BF16,)),
    "escapes_fp16": ("96x704 FP16 at 11 bpp: fields beyond the tables' symbol range, coded as escapes",
                     12, 11.0, (W.FP16, W.F32)),
    "int8_rows": ("64x512 INT8 rows scaled to +-127 at 3 bpp", 12, 3.0, (W.INT8, W.BF16)),
}


def matrix(name: str) -> W.Matrix:
    """The input of a case (container bit patterns)."""
    if name.startswith("small_bf16"):
        return W.small()
    if name == "ragged_bf16":
        g = np.random.Generator(np.random.PCG64(2037))
        return W.Matrix(W.to_bf16_bits(g.normal(0, 0.02, (37, 203))), W.BF16, 3.5)
    if name == "escapes_fp16":
        g = np.random.Generator(np.random.PCG64(2096))
        return W.Matrix(W.to_fp16_bits(g.normal(0, 0.02, (96, 704))), W.FP16, 11.0)
    if name == "int8_rows":
        return W.int8(rows=64, cols=512, target_bpp=3.0)
    raise KeyError(name)
