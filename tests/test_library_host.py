"""Host-side checks of the C-ABI library (no GPU needed).

* the library loads and exports every entry point include/entropack.h declares;
* the library's host encoder and the oracle's encoder, written independently from the same
  format description, produce byte-identical blobs, and the oracle decodes library blobs (one of
  the two cross directions; the other runs on the GPU);
* blob validation rejects corrupt bytes; argument errors map to their ep_status codes;
* the bytes do not depend on the encoder's thread count.
"""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import oracle
import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def ep():
    from dit_weight_compression_b200 import build
    build.build()
    import dit_weight_compression_b200 as ep
    return ep


def test_library_exports_every_declared_symbol(ep):
    header = open(os.path.join(ROOT, "include", "entropack.h")).read()
    declared = set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(ep_\w+)\s*\(", header, re.M))
    assert {"ep_compress", "ep_decompress", "ep_actual_bpp"} <= declared
    lib = ctypes.CDLL(ep.LIB_PATH)
    for name in sorted(declared):
        assert hasattr(lib, name), name
    assert declared == set(ep.SIGNATURES), declared ^ set(ep.SIGNATURES)


def _lib_blob(ep, m, **kw):
    cfg = ep.LatticeRANSConfig(m.target_bpp, **kw)
    return ep.compress(W.bits_to_torch(m.bits, m.dtype), cfg)


CASES = [
    ("small", lambda: W.small()),
    ("square", lambda: W.square(rows=512, cols=1024)),
    ("dit", lambda: W.dit(4, scale_down=8)),
    ("sweep0.5", lambda: W.sweep(0.5, rows=128, cols=1376)),
    ("sweep11", lambda: W.sweep(11.0, rows=64, cols=1376)),
    ("large", lambda: W.large(0, rows=256, cols=1024)),
    ("int8", lambda: W.int8(rows=256, cols=1024)),
]


@pytest.mark.parametrize("pb", [12, 10])
@pytest.mark.parametrize("name,make", CASES, ids=[c[0] for c in CASES])
def test_library_blob_equals_oracle_blob(ep, name, make, pb):
    m = make()
    lb = _lib_blob(ep, m, prob_bits=pb).to_bytes()
    ob = oracle.compress(m.bits, m.dtype, m.target_bpp, prob_bits=pb)
    assert lb == ob
    assert oracle.blob_info(lb)["prob_bits"] == pb


@pytest.mark.parametrize("name,make", [CASES[1], CASES[2], CASES[4], ("ragged", lambda: W.small(rows=37, cols=203))],
                         ids=["square", "dit", "sweep11", "ragged"])
def test_rd_refined_blob_equals_oracle_blob(ep, name, make):
    """The optional per-row rate-distortion refinement: library and oracle blobs byte-identical,
    and the thread count does not change the bytes."""
    m = make()
    pb = 10 if name == "dit" else 12
    ob = oracle.compress(m.bits, m.dtype, m.target_bpp, rd_refine=True, prob_bits=pb)
    for threads in (1, 5):
        cfg = ep.LatticeRANSConfig(m.target_bpp, num_threads=threads, rd_refine=True, prob_bits=pb)
        lb = ep.compress(W.bits_to_torch(m.bits, m.dtype), cfg).to_bytes()
        assert lb == ob


@pytest.mark.parametrize("shape", [(1, 1), (3, 13), (7, 9), (33, 7), (5, 1000), (2, 4096)])
@pytest.mark.parametrize("dtype", [W.BF16, W.FP16, W.E4M3, W.F32, W.INT8])
def test_ragged_and_containers_equal_oracle(ep, shape, dtype):
    g = np.random.Generator(np.random.PCG64(shape[0] * 7919 + shape[1] * 31 + dtype))
    x = g.normal(0, 0.05, shape)
    if dtype == W.INT8:
        x = x * 1000.0                                  # integers spread over the int8 range
    if dtype == W.E4M3:
        bits = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    else:
        bits = W._store(x, dtype)
    m = W.Matrix(bits, dtype, 4.0)
    lb = _lib_blob(ep, m).to_bytes()
    ob = oracle.compress(m.bits, m.dtype, m.target_bpp)
    assert lb == ob
    # the oracle decodes the library's blob and restores the shape
    out = oracle.decompress(lb)
    assert out.shape == shape


def test_oracle_decodes_library_blob_with_explicit_steps(ep):
    m = W.square(rows=300, cols=520)
    for S in (1, 3, 16, 100):
        c = _lib_blob(ep, m, steps_per_tile=S)
        b = c.to_bytes()
        assert oracle.blob_info(b)["S"] == S
        assert b == oracle.compress(m.bits, m.dtype, m.target_bpp, steps_per_tile=S)
        f = oracle.decode_fields(b)
        assert f.shape == (300 * 65, 9)


def test_thread_count_does_not_change_bytes(ep):
    m = W.square(rows=700, cols=512)
    ref = _lib_blob(ep, m, num_threads=1).to_bytes()
    for th in (2, 3, 8, 17):
        assert _lib_blob(ep, m, num_threads=th).to_bytes() == ref


def test_actual_bpp_and_info(ep):
    m = W.small(rows=100, cols=200)
    c = _lib_blob(ep, m)
    assert c.actual_bpp == 8.0 * len(c.to_bytes()) / (100 * 200)
    assert c.shape == (100, 200) and c.dtype == torch.bfloat16
    assert c.info.n_vectors == 100 * 25
    assert c.info.scale == oracle.blob_info(c.to_bytes())["scale"]


def test_roundtrip_bytes(ep):
    m = W.small()
    c = _lib_blob(ep, m)
    c2 = ep.CompressedTensor.from_bytes(c.to_bytes())
    assert c2.to_bytes() == c.to_bytes() and c2.shape == c.shape


def _corrupt(b: bytes, off: int, val: bytes) -> bytes:
    return b[:off] + val + b[off + len(val):]


def test_corrupt_blobs_rejected(ep):
    b = _lib_blob(ep, W.small()).to_bytes()
    bad = [
        b[:79],                                            # truncated header
        _corrupt(b, 0, b"EPK2"),                           # magic
        _corrupt(b, 4, b"\x01\x00"),                       # version (1: 12-bit totals)
        _corrupt(b, 6, b"\x09"),                           # dtype
        _corrupt(b, 7, b"\x7e"),                           # alphabet
        b[:-16],                                           # size mismatch
        _corrupt(b, 24, (1).to_bytes(4, "little")),        # S inconsistent with n_tiles
        _corrupt(b, 48, (81).to_bytes(8, "little")),       # misaligned table section
        _corrupt(b, 80, (1023).to_bytes(2, "little")),     # joint (coset, f1) table off 1024
    ]
    off_offs = int.from_bytes(b[64:72], "little")
    bad.append(_corrupt(b, off_offs + 4, (3).to_bytes(4, "little")))   # tile shorter than its header
    for i, x in enumerate(bad):
        with pytest.raises(ep.EPError) as e:
            ep.CompressedTensor.from_bytes(x)
        assert e.value.code == -5, i


def test_argument_errors(ep):
    t = torch.zeros((4, 8), dtype=torch.bfloat16)
    for bad in (0.0, 0.0009, 11.5, float("nan"), float("inf")):
        with pytest.raises((ep.EPError, ValueError)):
            ep.compress(t, bad)
    with pytest.raises(ep.EPError) as e:
        ep.compress(torch.zeros((0, 8), dtype=torch.bfloat16), 3.0)
    assert e.value.code == -3
    x = torch.zeros((4, 8), dtype=torch.bfloat16)
    x[1, 2] = float("nan")
    with pytest.raises(ep.EPError) as e:
        ep.compress(x, 3.0)
    assert e.value.code == -4
    # raw C call with an unknown dtype
    view = ep.EpTensor(t.data_ptr(), -1, 9, 4, 8, 8)
    h = ctypes.c_void_p()
    assert ep.lib().ep_compress(ctypes.byref(view), 3.0, ctypes.byref(h)) == -2
    view = ep.EpTensor(t.data_ptr(), -1, 1, 4, 8, 7)
    assert ep.lib().ep_compress(ctypes.byref(view), 3.0, ctypes.byref(h)) == -1
    assert ep.lib().ep_actual_bpp(None) == -1.0


def test_strided_host_input(ep):
    m = W.square(rows=64, cols=256)
    big = torch.zeros((64, 300), dtype=torch.bfloat16)
    big[:, :256] = W.bits_to_torch(m.bits, m.dtype)
    c = ep.compress(big[:, :256], 4.0)
    assert c.to_bytes() == oracle.compress(m.bits, m.dtype, 4.0)
