"""Every kernel variant the launch rule can pick, against the oracle on every tile.

A decode launch picks the layout of its shared-memory tables and its CTA width from the blob's tile
count, its largest tile and the SM count. The blobs here are sized to reach each (layout, width)
pair the rule uses: layouts 14, 13, 15, 11, 12 (12-bit totals) and 10 (10-bit totals), CTAs of 16,
20, 24 and 32 warps. For each one the test asserts that shape through ep_decode_shape, decodes, and
compares every element with the oracle's tile-parallel decode.

Tile sizes (i.i.d. N(0, 0.02^2) BF16, 8192 columns), largest: 4.0 bpp with S = 16 about 2.2 KB,
with S = 32 about 4064 B,
4.25 bpp with S = 32 4320 B, 2.5 bpp with S = 64 5088 B, 2.9 bpp 5904 B, 3.5 bpp 7136 B, 4.0 bpp
8144 B and 4.3 bpp 8768 B. Tile counts are multiples of the SM count, so the cases hold on any
GPU.
"""
import numpy as np
import pytest
import torch

import oracle_parallel
import workloads as W

pytestmark = pytest.mark.gpu

# (frequency-total bits, target bpp, S, tiles per SM, expected (layout, CTA warps))
CASES = [
    (12, 4.0, 32, 12, (14, 16)),   # tiles <= 4432 B: one round in 16-warp CTAs
    (12, 2.5, 64, 12, (13, 16)),   # 5 KB tiles: too large for layout 14
    (12, 4.0, 32, 18, (13, 20)),   # one round needs 20 warps: layout 13 has room for them
    (12, 3.5, 64, 12, (15, 16)),   # 7.1 KB tiles: too large for layout 13
    (12, 4.0, 64, 4, (11, 16)),    # 8 KB tiles: too large for layout 15
    (12, 4.3, 64, 4, (12, 16)),    # 8.7 KB tiles: layout 12's 16-warp buffers only
    (12, 2.5, 64, 18, (15, 20)),   # 5 KB tiles, one round in 20 warps
    (12, 2.9, 64, 18, (11, 20)),   # 5.9 KB tiles: too large for layout 15's 20-warp buffers
    (12, 3.5, 64, 18, (12, 20)),   # 7.1 KB tiles: too large for layout 11's 20-warp buffers
    (12, 4.0, 32, 22, (15, 24)),
    (12, 2.5, 64, 22, (11, 24)),   # 5 KB tiles: too large for layout 15's 24-warp buffers
    (12, 2.9, 64, 22, (12, 24)),   # 5.9 KB tiles: too large for layout 11's 24-warp buffers
    (12, 4.0, 16, 28, (15, 32)),   # 2.2 KB tiles
    (12, 4.0, 32, 28, (11, 32)),   # 4 KB tiles: too large for layout 15's 32-warp buffers
    (12, 4.25, 32, 28, (12, 32)),  # 4.3 KB tiles: too large for layout 11's 32-warp buffers
    (10, 4.0, 32, 12, (10, 16)),
    (10, 4.0, 32, 18, (10, 20)),
    (10, 4.0, 32, 22, (10, 24)),
    (10, 4.0, 32, 28, (10, 32)),
]


@pytest.fixture(scope="module")
def ep():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dit_weight_compression_b200 import build
    build.build()
    import dit_weight_compression_b200 as ep
    return ep


@pytest.mark.parametrize("pb,rate,S,per_sm,shape", CASES, ids=[f"L{c[4][0]}x{c[4][1]}" for c in CASES])
def test_every_launch_shape_matches_oracle(ep, pb, rate, S, per_sm, shape):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    cols = 8192
    rows = per_sm * sms * (32 * S) // (cols // 8)      # whole tiles: 32 S vectors, cols / 8 per row
    g = np.random.Generator(np.random.PCG64(pb * 1000 + per_sm * 10 + S))
    bits = W.to_bf16_bits(g.normal(0, 0.02, (rows, cols)))
    c = ep.compress(W.bits_to_torch(bits, W.BF16).cuda(), ep.LatticeRANSConfig(rate, steps_per_tile=S, prob_bits=pb))
    assert c.info.n_tiles == per_sm * sms
    assert ep.decode_shape(c) == shape
    out = ep.decompress(c)
    torch.cuda.synchronize()
    ep.decode_status(c)
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    want = oracle_parallel.decode(c.to_bytes())
    assert np.array_equal(got, want)
