"""The golden digests (tests/golden/oracle_digests.json, written from the oracle by
tests/golden/make_golden.py): exact bytes of blobs and decodes for small seeded cases.

Host: the oracle still writes and decodes those bytes, and the library's host encoder writes the
same blob. GPU: the library's GPU encoder writes the same blob, and the CUDA decode of it gives
the same output bytes in every listed container and in the row-scaled FP8 container.
"""
import hashlib
import json
import os
import sys

import numpy as np
import pytest
import torch

import oracle
import workloads as W

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "golden"))
from cases import CASES, matrix  # noqa: E402

GOLDEN = json.load(open(os.path.join(HERE, "golden", "oracle_digests.json")))["cases"]
NAME_TO_DTYPE = {v: k for k, v in W.DTYPE_NAME.items()}
TORCH = {W.BF16: torch.bfloat16, W.FP16: torch.float16, W.E4M3: torch.float8_e4m3fn, W.F32: torch.float32,
         W.INT8: torch.int8}


def sha(a) -> str:
    return hashlib.sha256(bytes(a) if isinstance(a, (bytes, bytearray)) else np.ascontiguousarray(a).tobytes()).hexdigest()


def test_every_case_has_a_digest():
    assert set(GOLDEN) == set(CASES)


@pytest.mark.parametrize("name", sorted(CASES))
def test_oracle_reproduces_the_digests(name):
    g = GOLDEN[name]
    m = matrix(name)
    blob = oracle.compress(m.bits, m.dtype, g["target_bpp"], prob_bits=g["prob_bits"])
    assert len(blob) == g["blob_bytes"] and sha(blob) == g["blob_sha256"]
    for dn, digest in g["decoded_sha256"].items():
        assert sha(oracle.decompress(blob, NAME_TO_DTYPE[dn])) == digest, dn
    pay, sig = oracle.decompress_rowscaled(blob)
    assert sha(pay) == g["rowscaled_payload_sha256"]
    assert sha(np.asarray(sig, np.float32)) == g["rowscaled_sigma_sha256"]


@pytest.fixture(scope="module")
def ep():
    from dit_weight_compression_b200 import build
    build.build()
    import dit_weight_compression_b200 as ep
    return ep


@pytest.mark.parametrize("name", sorted(CASES))
def test_library_host_encoder_writes_the_golden_blob(ep, name):
    g = GOLDEN[name]
    m = matrix(name)
    c = ep.compress(W.bits_to_torch(m.bits, m.dtype), ep.LatticeRANSConfig(g["target_bpp"], prob_bits=g["prob_bits"]))
    assert sha(c.to_bytes()) == g["blob_sha256"]


@pytest.mark.gpu
@pytest.mark.parametrize("name", sorted(CASES))
def test_gpu_encoder_and_decoder_match_the_digests(ep, name):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    g = GOLDEN[name]
    m = matrix(name)
    c = ep.compress(W.bits_to_torch(m.bits, m.dtype).cuda(),
                    ep.LatticeRANSConfig(g["target_bpp"], prob_bits=g["prob_bits"]))
    assert sha(c.to_bytes()) == g["blob_sha256"]
    for dn, digest in g["decoded_sha256"].items():
        out = ep.decompress(c, dtype=TORCH[NAME_TO_DTYPE[dn]])
        torch.cuda.synchronize()
        ep.decode_status(c)
        assert sha(out.contiguous().view(torch.uint8).cpu().numpy()) == digest, dn
    pay, sig = ep.decompress_fp8_rowscaled(c)
    torch.cuda.synchronize()
    assert sha(pay.contiguous().view(torch.uint8).cpu().numpy()) == g["rowscaled_payload_sha256"]
    assert sha(sig.cpu().numpy()) == g["rowscaled_sigma_sha256"]
