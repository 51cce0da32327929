"""Seeded synthetic weight matrices shaped like the codec's workloads.

This module only draws random numbers and stores them in a container dtype; it holds none of
the codec's arithmetic.  Both the oracle side (tests, CPU baseline) and the CUDA side (tests,
benchmark) take their inputs from here, so both read identical bytes.

Every matrix is drawn in float64 with ``numpy.random.Generator(PCG64(seed))`` and then rounded
to its container: BF16 by round-to-nearest-even through float32, FP16 by numpy's float64 ->
float16 cast (round-to-nearest-even).  Seeds are ``1000 + workload number``; matrix j of a
workload uses ``seed + j``.

Workloads (stand-ins for the pages' Z-Image-Turbo linear layers, whose weights are not
available; shapes follow DiT / transformer linear layers):

1. ``small``   256 x 256 BF16, i.i.d. N(0, 0.02^2), target 3.5 bits per element.
2. ``square``  4096 x 4096 BF16, row r i.i.d. N(0, sigma_r^2), sigma_r log-uniform in
               [0.005, 0.05], target 4.0.
3. ``dit``     four 3072 x 3072, one 3072 x 8192 and one 8192 x 3072 BF16 matrices, Student-t
               (nu = 5) scaled to std 0.02, 1% of rows (seeded permutation) scaled x10,
               target 2.5.
4. ``sweep``   4096 x 11008 FP16, i.i.d. N(0, 0.02^2), targets 0.5, 2.0, 3.5, 6.0, 11.0.
5. ``large``   four 28672 x 8192 BF16, N(0, 0.015^2) times per-column scales log-uniform in
               [0.5, 2], target 4.0; decoded to BF16 and to FP8 E4M3.
6. ``int8``    1024 x 4096 INT8 (the integer container): rows N(0, sigma_r^2), sigma_r
               log-uniform in [0.005, 0.05], each row scaled by 127 / its absmax and rounded to
               the nearest integer, target 3.0.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

BF16, FP16, E4M3, F32, INT8 = 1, 2, 3, 4, 5
DTYPE_NAME = {BF16: "bf16", FP16: "fp16", E4M3: "fp8_e4m3", F32: "fp32", INT8: "int8"}


@dataclass(frozen=True)
class Matrix:
    bits: np.ndarray     # rows x cols array of container bit patterns (uint16 / uint8 / uint32)
    dtype: int           # container code: 1 BF16, 2 FP16, 3 E4M3, 4 FP32, 5 INT8
    target_bpp: float

    @property
    def shape(self):
        return self.bits.shape


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float64 -> float32 (numpy cast, nearest-even) -> BF16 bit patterns (nearest-even)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def to_fp16_bits(x: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(x, np.float64).astype(np.float16).view(np.uint16)


def _store(x: np.ndarray, dtype: int) -> np.ndarray:
    if dtype == BF16:
        return to_bf16_bits(x)
    if dtype == FP16:
        return to_fp16_bits(x)
    if dtype == F32:
        return np.ascontiguousarray(x, np.float32).view(np.uint32)
    if dtype == INT8:  # nearest integer (ties to even), saturated
        return np.clip(np.rint(x), -128, 127).astype(np.int8).view(np.uint8)
    raise ValueError(dtype)


def _rng(workload: int, j: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(1000 + workload + j))


def small(rows: int = 256, cols: int = 256) -> Matrix:
    g = _rng(1)
    return Matrix(_store(g.standard_normal((rows, cols)) * 0.02, BF16), BF16, 3.5)


def square(rows: int = 4096, cols: int = 4096) -> Matrix:
    g = _rng(2)
    sigma = np.exp(g.uniform(np.log(0.005), np.log(0.05), size=(rows, 1)))
    return Matrix(_store(g.standard_normal((rows, cols)) * sigma, BF16), BF16, 4.0)


DIT_SHAPES = [(3072, 3072)] * 4 + [(3072, 8192), (8192, 3072)]


def dit(j: int, scale_down: int = 1) -> Matrix:
    rows, cols = DIT_SHAPES[j]
    rows, cols = rows // scale_down, cols // scale_down
    g = _rng(3, j)
    x = g.standard_t(5.0, size=(rows, cols)) * (0.02 / np.sqrt(5.0 / 3.0))
    hot = g.permutation(rows)[: int(round(0.01 * rows))]
    x[hot] *= 10.0
    return Matrix(_store(x, BF16), BF16, 2.5)


SWEEP_RATES = [0.5, 2.0, 3.5, 6.0, 11.0]


def sweep(target_bpp: float, rows: int = 4096, cols: int = 11008) -> Matrix:
    g = _rng(4)
    return Matrix(_store(g.standard_normal((rows, cols)) * 0.02, FP16), FP16, float(target_bpp))


def large(j: int, rows: int = 28672, cols: int = 8192) -> Matrix:
    g = _rng(5, j)
    colscale = np.exp(g.uniform(np.log(0.5), np.log(2.0), size=(1, cols)))
    x = g.standard_normal((rows, cols)) * 0.015 * colscale
    return Matrix(_store(x, BF16), BF16, 4.0)


def int8(rows: int = 1024, cols: int = 4096, target_bpp: float = 3.0) -> Matrix:
    """Integer weights as an INT8 checkpoint stores them: rows N(0, sigma_r^2) with sigma_r
    log-uniform in [0.005, 0.05], each row divided by its own absmax / 127 and rounded."""
    g = _rng(6)
    sigma = np.exp(g.uniform(np.log(0.005), np.log(0.05), size=(rows, 1)))
    x = g.standard_normal((rows, cols)) * sigma
    x = x / (np.abs(x).max(axis=1, keepdims=True) / 127.0)
    return Matrix(_store(x, INT8), INT8, target_bpp)


def bits_to_torch(bits: np.ndarray, dtype: int):
    """A torch CPU tensor of the container dtype sharing the bit patterns."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits))
    if dtype == BF16:
        return t.view(torch.bfloat16)
    if dtype == FP16:
        return t.view(torch.float16)
    if dtype == E4M3:
        return t.view(torch.float8_e4m3fn)
    if dtype == F32:
        return t.view(torch.float32)
    if dtype == INT8:
        return t.view(torch.int8)
    raise ValueError(dtype)
