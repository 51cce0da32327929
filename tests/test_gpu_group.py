"""Grouped decode (ep_decompress_group) through the C ABI.

One launch (per 32 blobs) decodes a set of blobs, each CTA working on one blob's tiles with that
blob's table.  The bar is the single-blob bar: every element bit-identical to the oracle's decode
of the same blob (and so to ep_decompress), for every container, on the shapes of a DiT block's
linear layers and on sets that mix tile lengths, escapes, ragged columns and strided outputs.
"""
import numpy as np
import pytest
import torch

import oracle
import oracle_parallel
import workloads as W

pytestmark = pytest.mark.gpu

TORCH = {W.BF16: torch.bfloat16, W.FP16: torch.float16, W.E4M3: torch.float8_e4m3fn, W.F32: torch.float32,
         W.INT8: torch.int8}
NP = {W.BF16: np.uint16, W.FP16: np.uint16, W.E4M3: np.uint8, W.F32: np.uint32, W.INT8: np.uint8}


@pytest.fixture(scope="module")
def ep():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dit_weight_compression_b200 import build
    build.build()
    import dit_weight_compression_b200 as ep
    return ep


def _bits(t: torch.Tensor, dtype: int) -> np.ndarray:
    v = {1: torch.int16, 2: torch.int16, 3: torch.uint8, 4: torch.int32, 5: torch.uint8}[dtype]
    return t.contiguous().view(v).cpu().numpy().view(NP[dtype])


def _compress(ep, m: W.Matrix, target=None, **kw):
    cfg = ep.LatticeRANSConfig(target or m.target_bpp, **kw)
    return ep.compress(W.bits_to_torch(m.bits, m.dtype), cfg)


def _status_all(ep, comps):
    torch.cuda.synchronize()
    for c in comps:
        ep.decode_status(c)


def test_group_dit_block_equals_single_decodes(ep):
    """The six linear layers of a DiT block (four 3072x3072, 3072x8192, 8192x3072; Student-t
    weights with hot rows) at 2.5 bpp, decoded in one launch: bit-identical to six ep_decompress
    calls and to the oracle's decode of every tile."""
    comps = [_compress(ep, W.dit(j)) for j in range(len(W.DIT_SHAPES))]
    outs = ep.decompress_group(comps)
    _status_all(ep, comps)
    for c, o in zip(comps, outs):
        single = ep.decompress(c)
        torch.cuda.synchronize()
        ep.decode_status(c)
        assert o.shape == single.shape and o.dtype == torch.bfloat16
        assert torch.equal(o.view(torch.int16), single.view(torch.int16))
        # and against the oracle, every tile
        assert np.array_equal(_bits(o, W.BF16), oracle_parallel.decode(c.to_bytes(), "values", W.BF16))


def _mixed_set(ep):
    """Blobs that take every variant of the kernel: tile lengths from 16 to 256 steps, an 11-bpp
    blob with escape words, ragged columns (element stores), a one-tile matrix, rows of fewer
    than 32 vectors, FP16 and BF16 inputs, 12-bit and 10-bit frequency totals."""
    specs = [
        (W.small(), None, {}),
        (W.square(rows=192, cols=1024), 4.0, {"steps_per_tile": 16}),
        (W.sweep(11.0, rows=48, cols=1000), None, {}),
        (W.sweep(0.5, rows=64, cols=1001), None, {}),
        (W.square(rows=8, cols=8), 4.0, {}),
        (W.dit(4, scale_down=8), None, {"steps_per_tile": 256}),
        (W.square(rows=300, cols=40), 3.0, {}),
        # 10-bit totals: the call splits the set into one launch per total width
        (W.square(rows=160, cols=768), 4.0, {"prob_bits": 10}),
        (W.sweep(11.0, rows=40, cols=704), None, {"prob_bits": 10}),
    ]
    out = []
    for m, t, kw in specs:
        c = _compress(ep, m, t, **kw)
        out.append((m, c, c.to_bytes()))
    return out


@pytest.mark.parametrize("dtype", [W.BF16, W.FP16, W.E4M3, W.F32, W.INT8])
def test_group_mixed_set_vs_oracle(ep, dtype):
    mixed = _mixed_set(ep)
    comps = [c for _, c, _ in mixed]
    assert any(c.info.n_tiles == 1 for c in comps)
    outs = ep.decompress_group(comps, dtype=TORCH[dtype])
    _status_all(ep, comps)
    for (m, c, blob), o in zip(mixed, outs):
        assert np.array_equal(_bits(o, dtype), oracle.decompress(blob, dtype))


def test_group_more_blobs_than_one_launch_holds(ep):
    """40 blobs: two launches (32 + 8); every blob decoded as the oracle decodes it."""
    mats = [W.square(rows=16 + j, cols=64 + 8 * (j % 5)) for j in range(40)]
    comps = [_compress(ep, m, 3.0) for m in mats]
    outs = ep.decompress_group(comps)
    _status_all(ep, comps)
    for c, o in zip(comps, outs):
        assert np.array_equal(_bits(o, W.BF16), oracle.decompress(c.to_bytes(), W.BF16))


def test_group_strided_outputs_and_repeated_blob(ep):
    """Outputs that are column windows of wider tensors (row stride > cols, aligned and
    misaligned), and the same blob twice in one call."""
    m = W.square(rows=64, cols=512)
    c = _compress(ep, m, 4.0)
    ref = oracle.decompress(c.to_bytes(), W.BF16)
    big = torch.zeros((64, 520), dtype=torch.bfloat16, device="cuda")
    big2 = torch.zeros((64, 515), dtype=torch.bfloat16, device="cuda")
    ep.decompress_group([c, c], outs=[big[:, :512], big2[:, 1:513]])
    _status_all(ep, [c])
    assert np.array_equal(_bits(big[:, :512], W.BF16), ref)
    assert np.array_equal(_bits(big2[:, 1:513], W.BF16), ref)
    assert torch.count_nonzero(big[:, 512:]) == 0 and torch.count_nonzero(big2[:, 0]) == 0


def test_group_corrupt_member_reported_alone(ep):
    """A blob whose tile payloads are damaged (it still passes host validation) is flagged by its
    own status word; the other blobs of the launch decode correctly."""
    good = [_compress(ep, W.square(rows=128, cols=1024), 4.0), _compress(ep, W.small())]
    b = bytearray(_compress(ep, W.square(rows=128, cols=1024), 4.0).to_bytes())
    off_stream = int.from_bytes(b[72:80], "little")
    for pos in (off_stream + 200, off_stream + 3000, len(b) - 40):
        b[pos] ^= 0x5A
    bad = ep.CompressedTensor.from_bytes(bytes(b))
    outs = ep.decompress_group([good[0], bad, good[1]])
    torch.cuda.synchronize()
    with pytest.raises(ep.EPError) as e:
        ep.decode_status(bad)
    assert e.value.code == -5
    for c, o in zip(good, (outs[0], outs[2])):
        ep.decode_status(c)
        assert np.array_equal(_bits(o, W.BF16), oracle.decompress(c.to_bytes(), W.BF16))


def test_group_argument_errors(ep):
    a = _compress(ep, W.small())
    b = _compress(ep, W.square(rows=16, cols=64), 3.0)
    assert ep.decompress_group([]) == []
    with pytest.raises(ep.EPError) as e:       # outputs of two dtypes
        ep.decompress_group([a, b], outs=[torch.empty(a.shape, dtype=torch.bfloat16, device="cuda"),
                                          torch.empty(b.shape, dtype=torch.float16, device="cuda")])
    assert e.value.code == -2
    with pytest.raises(ep.EPError) as e:       # a wrong shape
        ep.decompress_group([a, b], outs=[torch.empty(a.shape, dtype=torch.bfloat16, device="cuda"),
                                          torch.empty((16, 72), dtype=torch.bfloat16, device="cuda")])
    assert e.value.code == -3
    with pytest.raises(ep.EPError) as e:       # host outputs are not accepted
        ep.decompress_group([a], outs=[torch.empty(a.shape, dtype=torch.bfloat16)])
    assert e.value.code == -1
