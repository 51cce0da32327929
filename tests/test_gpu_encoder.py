"""The encoder on the GPU (ep_compress of a CUDA tensor), through the C ABI.

The bar is byte identity: a CUDA tensor compressed on its GPU gives exactly the blob the oracle
writes for the same elements (and so exactly the host encoder's blob) -- for every container,
ragged and strided inputs, any tile length, escape-heavy rates and a forced scale.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ep():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dit_weight_compression_b200 import build
    build.build()
    import dit_weight_compression_b200 as ep
    return ep


def _gpu_blob(ep, m: W.Matrix, target=None, **kw) -> bytes:
    t = W.bits_to_torch(m.bits, m.dtype).cuda()
    return ep.compress(t, ep.LatticeRANSConfig(target or m.target_bpp, **kw)).to_bytes()


CASES = [
    ("small", lambda: W.small()),
    ("square", lambda: W.square(rows=1024, cols=2048)),
    ("dit", lambda: W.dit(4, scale_down=4)),
    ("sweep0.5", lambda: W.sweep(0.5, rows=256, cols=1376)),
    ("sweep11", lambda: W.sweep(11.0, rows=128, cols=1376)),
    ("large", lambda: W.large(0, rows=512, cols=2048)),
    ("int8", lambda: W.int8(rows=256, cols=1024)),
]


@pytest.mark.parametrize("pb", [12, 10])
@pytest.mark.parametrize("name,make", CASES, ids=[c[0] for c in CASES])
def test_gpu_encoder_equals_oracle(ep, name, make, pb):
    m = make()
    assert _gpu_blob(ep, m, prob_bits=pb) == oracle.compress(m.bits, m.dtype, m.target_bpp, prob_bits=pb)


def test_gpu_encoder_full_size_square(ep):
    """The 4096 x 4096 BF16 workload at 4 bpp: the GPU blob equals the host encoder's blob (the
    host encoder is byte-identical to the oracle on every case of the host suite)."""
    m = W.square()
    t = W.bits_to_torch(m.bits, m.dtype)
    host = ep.compress(t, ep.LatticeRANSConfig(4.0)).to_bytes()
    assert _gpu_blob(ep, m) == host


@pytest.mark.parametrize("shape", [(1, 1), (3, 13), (7, 9), (33, 7), (5, 1000), (2, 4096), (70, 37)])
@pytest.mark.parametrize("dtype", [W.BF16, W.FP16, W.E4M3, W.F32, W.INT8])
def test_gpu_encoder_ragged_and_containers(ep, shape, dtype):
    g = np.random.Generator(np.random.PCG64(shape[0] * 7919 + shape[1] * 31 + dtype))
    x = g.normal(0, 0.05, shape)
    if dtype == W.INT8:
        x = x * 1000.0
    if dtype == W.E4M3:
        bits = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    else:
        bits = W._store(x, dtype)
    m = W.Matrix(bits, dtype, 4.0)
    assert _gpu_blob(ep, m) == oracle.compress(m.bits, m.dtype, m.target_bpp)


@pytest.mark.parametrize("S", [1, 3, 16, 100, 1024])
def test_gpu_encoder_tile_lengths(ep, S):
    m = W.square(rows=300, cols=520)
    assert _gpu_blob(ep, m, steps_per_tile=S) == oracle.compress(m.bits, m.dtype, m.target_bpp, steps_per_tile=S)


def test_gpu_encoder_strided_input_and_forced_scale(ep):
    m = W.square(rows=128, cols=512)
    wide = torch.zeros((128, 640), dtype=torch.bfloat16, device="cuda")
    wide[:, 64:576] = W.bits_to_torch(m.bits, m.dtype).cuda()
    view = wide[:, 64:576]                                  # row stride 640
    got = ep.compress(view, ep.LatticeRANSConfig(4.0)).to_bytes()
    assert got == oracle.compress(m.bits, m.dtype, 4.0)
    got = ep.compress(view, ep.LatticeRANSConfig(4.0), scale=0.37).to_bytes()
    assert got == oracle.compress(m.bits, m.dtype, 4.0, scale=0.37)


def test_gpu_encoder_switches(ep):
    """host_encoder=True gives the same bytes; rd_refine runs on the host (same as the oracle's
    refined blob); the all-zero matrix; a non-finite element is rejected."""
    m = W.square(rows=64, cols=512)
    t = W.bits_to_torch(m.bits, m.dtype).cuda()
    a = ep.compress(t, ep.LatticeRANSConfig(4.0)).to_bytes()
    b = ep.compress(t, ep.LatticeRANSConfig(4.0, host_encoder=True)).to_bytes()
    assert a == b
    r = ep.compress(t, ep.LatticeRANSConfig(4.0, rd_refine=True)).to_bytes()
    assert r == oracle.compress(m.bits, m.dtype, 4.0, rd_refine=True)
    z = torch.zeros((16, 64), dtype=torch.bfloat16, device="cuda")
    assert ep.compress(z, 3.0).to_bytes() == oracle.compress(np.zeros((16, 64), np.uint16), W.BF16, 3.0)
    bad = t.clone()
    bad[5, 7] = float("inf")
    with pytest.raises(ep.EPError) as e:
        ep.compress(bad, 4.0)
    assert e.value.code == -4
