"""GPU parity: the CUDA decode against the oracle, through the C ABI.

Bars (per element):
  * fields (coset bit, f1..f8) bit-exact;
  * restored values within 1 ulp of the output container -- both sides compute the same IEEE
    sequence (fp32 product of the fp32 row scale and the exact lattice coordinate, then one
    round-to-nearest-even into the container), so the checks below require 0 ulp;
  * ||output - input|| / ||input|| equal to the oracle's to 1e-6.
Both cross directions: the GPU decodes oracle-encoded blobs, and the oracle decodes library-encoded
blobs (here at full size, tile-parallel on the host cores, and in the host suite).  Every element of
every full-size workload is compared.
"""
import ctypes

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
PBS = (12, 10)   # frequency totals: 12-bit (the format's choice, default) and 10-bit


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


def _ulp(a: np.ndarray, b: np.ndarray, dtype: int) -> np.ndarray:
    """Distance in units in the last place between two arrays of container bit patterns."""
    if dtype == W.INT8:
        return np.abs(a.view(np.int8).astype(np.int64) - b.view(np.int8).astype(np.int64))
    nb = {1: 16, 2: 16, 3: 8, 4: 32}[dtype]
    def key(x):
        x = x.astype(np.int64)
        sign = 1 << (nb - 1)
        return np.where(x & sign, -(x & (sign - 1)), x)
    return np.abs(key(a) - key(b))


def _rel_l2(bits, dtype, ref):
    x = oracle.dtype_to_f64(bits, dtype)
    return np.linalg.norm(x - ref) / np.linalg.norm(ref)


def _gpu_decode(ep, c, dtype=None, **kw):
    out = ep.decompress(c, dtype=TORCH[dtype] if dtype else None, **kw)
    torch.cuda.synchronize()
    ep.decode_status(c)
    return out


def _check_full(ep, blob: bytes, m: W.Matrix, out_dtypes=None):
    """Every field and every element against the oracle."""
    c = ep.CompressedTensor.from_bytes(blob)
    f_gpu = ep.decode_fields(c).cpu().numpy()
    ep.decode_status(c)
    assert np.array_equal(f_gpu, oracle.decode_fields(blob))
    ref = oracle.dtype_to_f64(m.bits, m.dtype)
    for dt in out_dtypes or [m.dtype]:
        g = _bits(_gpu_decode(ep, c, dt), dt)
        o = oracle.decompress(blob, dt)
        assert g.shape == o.shape
        assert _ulp(g, o, dt).max() <= 1
        assert np.array_equal(g, o)
        if dt != W.E4M3 and np.linalg.norm(ref) > 0:   # (an all-zero input has no relative error)
            assert abs(_rel_l2(g, dt, ref) - _rel_l2(o, dt, ref)) <= 1e-6
    return c


# ---------------------------------------------------------------------------------------------
# GPU decodes oracle-encoded blobs (cross direction 1), every element.
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("pb", PBS)
def test_small_oracle_blob_all_containers(ep, pb):
    m = W.small()
    blob = oracle.compress(m.bits, m.dtype, m.target_bpp, prob_bits=pb)
    assert oracle.blob_info(blob)["prob_bits"] == pb
    _check_full(ep, blob, m, [W.BF16, W.FP16, W.E4M3, W.F32, W.INT8])


def test_rd_refined_oracle_blob(ep):
    """A blob made with the per-row rate-distortion refinement (rows at different resolutions,
    the decode format unchanged) decodes as the oracle decodes it."""
    m = W.square(rows=512, cols=1024)
    blob = oracle.compress(m.bits, m.dtype, m.target_bpp, rd_refine=True)
    _check_full(ep, blob, m, [W.BF16, W.F32])


def test_int8_container_oracle_blob(ep):
    """An INT8 input (rows scaled to their absmax) restored as INT8 -- nearest integer, ties to
    even, saturated -- and, from the same blob, as BF16 and FP32."""
    m = W.int8()
    blob = oracle.compress(m.bits, m.dtype, m.target_bpp)
    assert oracle.blob_info(blob)["dtype"] == W.INT8
    c = _check_full(ep, blob, m, [W.INT8, W.BF16, W.F32])
    assert c.dtype == torch.int8


@pytest.mark.parametrize("pb", PBS)
def test_square_full_size_oracle_blob(ep, pb):
    m = W.square()
    blob = oracle.compress(m.bits, m.dtype, m.target_bpp, prob_bits=pb)
    _check_full(ep, blob, m)


@pytest.mark.parametrize("pb", PBS)
@pytest.mark.parametrize("S", [1, 2, 3, 16, 33, 1024])
def test_steps_per_tile_and_partial_tiles(ep, S, pb):
    m = W.square(rows=97, cols=1000)
    blob = oracle.compress(m.bits, m.dtype, 4.0, steps_per_tile=S, prob_bits=pb)
    _check_full(ep, blob, m, [W.BF16, W.F32])


@pytest.mark.parametrize("cols,S,pb", [(256, 5, 12), (512, 3, 10), (768, 3, 12), (768, 16, 10), (1280, 5, 12),
                                       (1536, 100, 12), (1792, 7, 10)])
def test_short_rows_tiles_starting_mid_row(ep, cols, S, pb):
    """Rows of 1 to 7 steps (a multiple of 32 vectors per row, so a warp's lanes change rows
    together) with tile lengths that are not multiples of the row length: tiles start and end
    inside rows, the row change falls anywhere in a tile's run of steps, the last tile is
    partial."""
    m = W.square(rows=41, cols=cols)
    blob = oracle.compress(m.bits, m.dtype, 4.0, steps_per_tile=S, prob_bits=pb)
    _check_full(ep, blob, m, [W.BF16, W.FP16, W.E4M3])


@pytest.mark.parametrize("pb", PBS)
@pytest.mark.parametrize("S,rate", [(1, 11.0), (2, 4.0), (1, 0.5)])
def test_many_tiles_per_warp(ep, S, rate, pb):
    """More tiles than resident warps (148 SMs x 32 warps), so warps decode several tiles one
    after another, each staged into the buffer the previous one used."""
    m = W.sweep(rate, rows=2400, cols=1024)
    blob = oracle.compress(m.bits, m.dtype, rate, steps_per_tile=S, prob_bits=pb)
    assert oracle.blob_info(blob)["n_tiles"] > 148 * 32
    _check_full(ep, blob, m)


@pytest.mark.parametrize("pb", PBS)
@pytest.mark.parametrize("shape", [(1, 1), (1, 8), (3, 13), (7, 9), (33, 7), (5, 1000), (17, 4100)])
def test_ragged_shapes(ep, shape, pb):
    g = np.random.Generator(np.random.PCG64(shape[0] * 1000 + shape[1]))
    m = W.Matrix(W.to_bf16_bits(g.normal(0, 0.02, shape)), W.BF16, 3.0)
    blob = oracle.compress(m.bits, m.dtype, m.target_bpp, prob_bits=pb)
    _check_full(ep, blob, m, [W.BF16, W.FP16, W.E4M3, W.F32, W.INT8])


@pytest.mark.parametrize("pb", PBS)
@pytest.mark.parametrize("rate", [0.5, 2.0, 11.0])
def test_rate_extremes_oracle_blob(ep, rate, pb):
    m = W.sweep(rate, rows=128, cols=1376)
    blob = oracle.compress(m.bits, m.dtype, rate, prob_bits=pb)
    _check_full(ep, blob, m)


@pytest.mark.parametrize("pb", PBS)
def test_degenerate_tables(ep, pb):
    # constant rows: lone symbols (q = M) in most contexts; a zero row; FP16 input
    g = np.random.Generator(np.random.PCG64(5))
    x = g.normal(0, 0.05, (64, 1)) * np.ones((1, 1024))
    x[3] = 0.0
    m = W.Matrix(W.to_fp16_bits(x), W.FP16, 4.0)
    blob = oracle.compress(m.bits, m.dtype, m.target_bpp, prob_bits=pb)
    _check_full(ep, blob, m)
    z = W.Matrix(W.to_bf16_bits(np.zeros((40, 64))), W.BF16, 1.0)
    blob = oracle.compress(z.bits, z.dtype, z.target_bpp, prob_bits=pb)
    _check_full(ep, blob, z)


def test_tiny_row_scales(ep):
    """Rows around 2^-135 (FP32 subnormals) give row scales below 2^-125, where any rewriting of
    alpha * y that scales alpha first (halving it, say) would round: the kernel's exact lattice
    coordinate times alpha, rounded once, must still equal the oracle's."""
    g = np.random.Generator(np.random.PCG64(11))
    x = g.normal(0, 1, (64, 256)) * 2.0 ** -135
    x[::2] *= 2.0 ** 100                                           # half the rows ordinary
    m = W.Matrix(np.ascontiguousarray(x, np.float32).view(np.uint32), W.F32, 4.0)
    blob = oracle.compress(m.bits, m.dtype, m.target_bpp)
    _check_full(ep, blob, m, [W.F32, W.BF16])


# ---------------------------------------------------------------------------------------------
# Library-encoded blobs at full workload sizes: every tile against the oracle, which decodes them
# tile-parallel on the host cores (cross direction 2: the oracle decodes library blobs).
# ---------------------------------------------------------------------------------------------

def _check_every_tile(ep, c, m: W.Matrix, out_dtypes=None, fields=True):
    blob = c.to_bytes()
    if fields:
        f_gpu = ep.decode_fields(c).cpu().numpy()
        ep.decode_status(c)
        assert np.array_equal(f_gpu, oracle_parallel.decode(blob, "fields"))
    ref = oracle.dtype_to_f64(m.bits, m.dtype)
    for dt in out_dtypes or [m.dtype]:
        g = _bits(_gpu_decode(ep, c, dt), dt)
        o = oracle_parallel.decode(blob, "values", dt)
        assert np.array_equal(g, o), dt
        if dt != W.E4M3:
            assert abs(_rel_l2(g, dt, ref) - _rel_l2(o, dt, ref)) <= 1e-6


def test_dit_set_full_size(ep):
    for j in range(len(W.DIT_SHAPES)):
        m = W.dit(j)
        c = ep.compress(W.bits_to_torch(m.bits, m.dtype), m.target_bpp)
        _check_every_tile(ep, c, m)


@pytest.mark.parametrize("rate", W.SWEEP_RATES)
def test_sweep_full_size(ep, rate):
    m = W.sweep(rate)
    c = ep.compress(W.bits_to_torch(m.bits, m.dtype), rate)
    _check_every_tile(ep, c, m)


def test_large_layer_full_size_bf16_and_fp8(ep):
    """The four 28672 x 8192 matrices of the large-layer stream, every tile: each decoded alone to
    BF16 and to the E4M3 container against the oracle, then all four in one grouped launch (the
    benchmark's path, with the table layout and CTA width the set's tile count gives) against
    the single decodes."""
    comps = []
    for j in range(4):
        m = W.large(j)
        c = ep.compress(W.bits_to_torch(m.bits, m.dtype), m.target_bpp)
        _check_every_tile(ep, c, m, [W.BF16, W.E4M3], fields=(j == 0))
        comps.append(c)
    for dt in (torch.bfloat16, torch.float8_e4m3fn):
        singles = [ep.decompress(c, dtype=dt) for c in comps]
        grouped = ep.decompress_group(comps, dtype=dt)
        torch.cuda.synchronize()
        for c in comps:
            ep.decode_status(c)
        for a, b in zip(singles, grouped):
            assert torch.equal(a.view(torch.uint8), b.view(torch.uint8)), dt
        del singles, grouped


# ---------------------------------------------------------------------------------------------
# Output layouts, streams, the end-to-end host path, and corruption reporting.
# ---------------------------------------------------------------------------------------------

def test_strided_and_misaligned_outputs(ep):
    m = W.square(rows=64, cols=512)
    blob = oracle.compress(m.bits, m.dtype, 4.0)
    c = ep.CompressedTensor.from_bytes(blob)
    ref = oracle.decompress(blob, W.BF16)
    big = torch.zeros((64, 520), dtype=torch.bfloat16, device="cuda")
    ep.decompress(c, out=big[:, :512])                      # row stride 520 (vector stores)
    big2 = torch.zeros((64, 515), dtype=torch.bfloat16, device="cuda")
    ep.decompress(c, out=big2[:, 1:513])                    # misaligned: element stores
    torch.cuda.synchronize()
    ep.decode_status(c)
    assert np.array_equal(_bits(big[:, :512], W.BF16), ref)
    assert np.array_equal(_bits(big2[:, 1:513], W.BF16), ref)
    assert torch.count_nonzero(big[:, 512:]) == 0 and torch.count_nonzero(big2[:, 0]) == 0


def test_host_output_path_matches_device_path(ep):
    m = W.square(rows=256, cols=1024)
    c = ep.compress(W.bits_to_torch(m.bits, m.dtype), 4.0)
    dev = _bits(_gpu_decode(ep, c), W.BF16)
    host = torch.empty((256, 1024), dtype=torch.bfloat16).pin_memory()
    ep.decompress(c, out=host)
    assert np.array_equal(_bits(host, W.BF16), dev)
    ep.decode_status(c)


@pytest.mark.parametrize("rows,cols,dtype,rate,pinned,pad", [
    (2048, 4096, W.BF16, 4.0, True, 0),     # 4 chunks; a tile is 2 rows, so every tile starts a row
    (4104, 4099, W.BF16, 4.0, True, 0),     # ragged rows: a row-aligned unit is 513 tiles, the last
                                            # chunk holds the 5 tiles left, the last one partial
    (3072, 3072, W.FP16, 2.5, False, 24),   # 3 tiles per row-aligned unit; pageable, strided output
])
def test_host_output_chunks_match_device_path(ep, rows, cols, dtype, rate, pinned, pad):
    """A host output of 8 MB or more comes back in chunks of whole rows, each downloaded while
    the next is uploaded and decoded: the bytes equal the device path's for every chunk geometry,
    and nothing outside the output's columns is written."""
    g = np.random.Generator(np.random.PCG64(rows * 7 + cols))
    x = g.normal(0, 0.02, (rows, cols))
    bits = W.to_bf16_bits(x) if dtype == W.BF16 else W.to_fp16_bits(x)
    c = ep.compress(W.bits_to_torch(bits, dtype), rate)
    ref = _bits(_gpu_decode(ep, c), dtype)
    tdt = TORCH[dtype]
    big = torch.full((rows, cols + pad), 7.0, dtype=tdt)
    if pinned:
        big = big.pin_memory()
    view = big[:, :cols]
    ep.decompress(c, out=view)
    ep.decode_status(c)
    assert np.array_equal(_bits(view, dtype), ref)
    if pad:
        assert torch.all(big[:, cols:] == 7.0)
    again = torch.empty((rows, cols), dtype=tdt).pin_memory()    # a second call reuses the staging
    ep.decompress(c, out=again)
    assert np.array_equal(_bits(again, dtype), ref)


def test_side_stream(ep):
    m = W.small()
    c = ep.compress(W.bits_to_torch(m.bits, m.dtype), m.target_bpp)
    s = torch.cuda.Stream()
    c.prepare(stream=s)
    with torch.cuda.stream(s):
        out = ep.decompress(c, stream=s)
    s.synchronize()
    assert np.array_equal(_bits(out, W.BF16), oracle.decompress(c.to_bytes()))


def test_corrupt_stream_reported_not_hung(ep):
    """Flip bits inside tile payloads (the blob still passes host validation): the kernel must
    finish, flag the status word, and leave the context usable."""
    m = W.square(rows=128, cols=1024)
    b = bytearray(ep.compress(W.bits_to_torch(m.bits, m.dtype), 4.0).to_bytes())
    off_stream = int.from_bytes(b[72:80], "little")
    for pos in (off_stream + 200, off_stream + 3000, len(b) - 40):
        b[pos] ^= 0x5A
    c = ep.CompressedTensor.from_bytes(bytes(b))
    out = ep.decompress(c)
    torch.cuda.synchronize()
    with pytest.raises(ep.EPError) as e:
        ep.decode_status(c)
    assert e.value.code == -5
    # the context still works and the status word was cleared
    good = ep.compress(W.bits_to_torch(m.bits, m.dtype), 4.0)
    ep.decompress(good)
    ep.decode_status(good)
    del out


def test_bounded_wait_gives_up_and_reports(ep):
    """A bulk-copy wait that can never complete (the barrier expects bytes no copy delivers) gives
    up after its short limit: the kernel ends, the status word reports the wait limit, and the
    context stays usable -- nothing faults or hangs."""
    m = W.small()
    c = ep.compress(W.bits_to_torch(m.bits, m.dtype), m.target_bpp)
    ref = _gpu_decode(ep, c)                  # also makes the blob's device copy
    L = ep.lib()
    rc = L.ep_decode_wait_probe(c.handle, 2000, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, L.ep_last_error()
    torch.cuda.synchronize()
    with pytest.raises(ep.EPError) as e:
        ep.decode_status(c)
    assert e.value.code == -5 and "wait limit" in str(e.value)
    again = _gpu_decode(ep, c)                # status cleared, decode still correct
    assert np.array_equal(_bits(again, W.BF16), _bits(ref, W.BF16))


def test_rel_l2_matches_oracle_usage_example(ep):
    """The pages' usage example: 256 x 256 BF16 N(0, 0.02^2) at 3.5 bpp; restored shape and
    dtype equal the input's; stored rate and relative L2 error as the oracle reports them."""
    m = W.small()
    t = W.bits_to_torch(m.bits, m.dtype).cuda()
    cfg = ep.LatticeRANSConfig(target_bpp=3.5)
    comp = ep.compress(t, cfg)
    restored = ep.decompress(comp, cfg)
    assert restored.shape == t.shape and restored.dtype == t.dtype
    rel = ((restored.float() - t.float()).norm() / t.float().norm()).item()
    blob = comp.to_bytes()
    rel_o = _rel_l2(oracle.decompress(blob), W.BF16, oracle.dtype_to_f64(m.bits, m.dtype))
    assert abs(rel - rel_o) <= 1e-6
    assert comp.actual_bpp == oracle.actual_bpp(blob)
