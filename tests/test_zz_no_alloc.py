"""The allocation-free decode entry point, ep_decompress_noalloc, through the C ABI.

Some callers cannot let a library allocate GPU memory: an inference runtime that lays out all
device memory ahead of time in its own arena, or code running where an allocation is forbidden
or would synchronise the device.  For them ep_decompress_noalloc takes the blob's bytes already
in device memory (their allocation, not the library's) and keeps the decode kernel's status word
in a fixed array inside the library instead of allocating one.

This file checks that entry point against the ordinary ep_decompress on the same blob, bit for
bit (the tolerance the parity tests use), on two calls in a row, for every kernel variant it can
launch: vector and element stores, blobs with and without escape symbols, each output container
and both frequency-total widths.  It also checks that the two calls leave the device's free memory
unchanged (after a first call has let the driver load the kernel variant), that a
corrupt tile is reported and the next clean call is not, and that a device buffer shorter than
the blob is refused.  It is named so that pytest collects it after every other test file.
"""
import ctypes
import struct

import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu

TORCH = {W.BF16: torch.bfloat16, W.FP16: torch.float16, W.E4M3: torch.float8_e4m3fn, W.F32: torch.float32,
         W.INT8: torch.int8}


@pytest.fixture(scope="module")
def ep():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dit_weight_compression_b200 import build
    build.build()
    import dit_weight_compression_b200 as ep
    return ep


def _bytes(t):
    return t.contiguous().view(torch.uint8).cpu().numpy()


def _noalloc(ep, comp, dev_blob, out, wait=1, nbytes=None):
    L = ep.lib()
    view = ep.tensor_view(out)
    n = dev_blob.numel() if nbytes is None else nbytes
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.ep_decompress_noalloc(comp.handle, ctypes.c_void_p(dev_blob.data_ptr()), n, ctypes.byref(view), s,
                                   wait)


def _two_calls_match(ep, comp, out_dtype, make_out):
    """Two allocation-free decodes in a row equal ep_decompress, with free memory unchanged.
    One call comes first, unchecked: the first launch of a kernel variant lets the CUDA driver
    load that kernel's code (lazy module loading), which can take device memory -- the driver's,
    not the library's -- so the memory check starts after it."""
    ref = make_out()
    ep.decompress(comp, out=ref)
    torch.cuda.synchronize()
    ep.decode_status(comp)
    dev_blob = torch.frombuffer(bytearray(comp.to_bytes()), dtype=torch.uint8).cuda()
    assert dev_blob.data_ptr() % 16 == 0
    outs = [make_out() for _ in range(2)]
    for o in outs:
        o.view(torch.uint8).fill_(0x7F)
    warm = make_out()
    assert _noalloc(ep, comp, dev_blob, warm) == 0, ep.lib().ep_last_error()
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    for o in outs:
        rc = _noalloc(ep, comp, dev_blob, o)
        assert rc == 0, ep.lib().ep_last_error()
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    for o in outs:
        assert np.array_equal(_bytes(o), _bytes(ref)), out_dtype
    assert free_after == free_before


@pytest.mark.parametrize("pb", [12, 10])
def test_noalloc_matches_decompress_twice(ep, pb):
    """BF16, vector stores, an escape-free blob; 12-bit and 10-bit frequency totals."""
    m = W.square(rows=1024, cols=2048)
    comp = ep.compress(W.bits_to_torch(m.bits, m.dtype), ep.LatticeRANSConfig(m.target_bpp, prob_bits=pb))
    _two_calls_match(ep, comp, W.BF16, lambda: torch.empty(comp.shape, dtype=torch.bfloat16, device="cuda"))


@pytest.mark.parametrize("rate", [3.5, 4.0, 4.3])
def test_noalloc_large_tiles(ep, rate):
    """Tiles of about 7.1, 8.1 and 8.8 KB (S = 64): too large for layout 13's buffers, so the
    allocation-free kernel takes layout 15 (the joint table and f2 direct), layout 11 (the joint
    table direct) and layout 12 (every symbol in two lookups), each with its tables built inside
    every CTA."""
    g = np.random.Generator(np.random.PCG64(int(rate * 100)))
    bits = W.to_bf16_bits(g.normal(0, 0.02, (256, 8192)))
    comp = ep.compress(W.bits_to_torch(bits, W.BF16), ep.LatticeRANSConfig(rate, steps_per_tile=64))
    _two_calls_match(ep, comp, W.BF16, lambda: torch.empty(comp.shape, dtype=torch.bfloat16, device="cuda"))


@pytest.mark.parametrize("dtype", [W.FP16, W.E4M3, W.F32, W.INT8])
def test_noalloc_escapes_every_container(ep, dtype):
    """An 11-bpp blob (most fields are escapes, so the escape kernel runs) in every container."""
    m = W.sweep(11.0, rows=96, cols=704)
    comp = ep.compress(W.bits_to_torch(m.bits, m.dtype), m.target_bpp)
    _two_calls_match(ep, comp, dtype, lambda: torch.empty(comp.shape, dtype=TORCH[dtype], device="cuda"))


@pytest.mark.parametrize("dtype", [W.BF16, W.E4M3])
def test_noalloc_element_stores(ep, dtype):
    """Outputs the vector stores cannot take: ragged columns, and a misaligned output pointer."""
    m = W.small(rows=37, cols=203)
    comp = ep.compress(W.bits_to_torch(m.bits, m.dtype), m.target_bpp)
    _two_calls_match(ep, comp, dtype, lambda: torch.empty(comp.shape, dtype=TORCH[dtype], device="cuda"))
    m2 = W.small(rows=40, cols=256)
    comp2 = ep.compress(W.bits_to_torch(m2.bits, m2.dtype), m2.target_bpp)

    def shifted():
        base = torch.empty(40 * 256 + 1, dtype=TORCH[dtype], device="cuda")
        return base[1:].view(40, 256)   # one element off the vector alignment

    _two_calls_match(ep, comp2, dtype, shifted)


def test_noalloc_corrupt_tile_then_clean_call(ep):
    """Flipped payload bytes inside one tile (offsets and headers intact) give EP_ERR_CORRUPT; the
    next call on intact bytes returns 0, because each call clears the shared status word."""
    m = W.square(rows=256, cols=1024)
    comp = ep.compress(W.bits_to_torch(m.bits, m.dtype), m.target_bpp)
    blob = comp.to_bytes()
    off_offsets, off_stream = struct.unpack_from("<QQ", blob, 64)   # header: tile-offset, stream offsets
    off = off_stream + 16 * struct.unpack_from("<I", blob, off_offsets + 4)[0]   # start of tile 1
    bad = bytearray(blob)
    for k in range(off + 200, off + 260):      # inside tile 1's regions, past its 160-byte header
        bad[k] ^= 0x5A
    out = torch.empty(comp.shape, dtype=torch.bfloat16, device="cuda")
    dev_bad = torch.frombuffer(bad, dtype=torch.uint8).cuda()
    dev_good = torch.frombuffer(bytearray(blob), dtype=torch.uint8).cuda()
    assert _noalloc(ep, comp, dev_bad, out) == -5
    assert b"corrupt" in ep.lib().ep_last_error()
    assert _noalloc(ep, comp, dev_good, out) == 0
    ref = ep.decompress(comp)
    torch.cuda.synchronize()
    assert np.array_equal(_bytes(out), _bytes(ref))


def test_noalloc_rejects_bad_arguments(ep):
    m = W.small()
    comp = ep.compress(W.bits_to_torch(m.bits, m.dtype), m.target_bpp)
    dev_blob = torch.frombuffer(bytearray(comp.to_bytes()), dtype=torch.uint8).cuda()
    out = torch.empty(comp.shape, dtype=torch.bfloat16, device="cuda")
    view = ep.tensor_view(out)
    L = ep.lib()
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    n = dev_blob.numel()
    # misaligned device bytes
    rc = L.ep_decompress_noalloc(comp.handle, ctypes.c_void_p(dev_blob.data_ptr() + 8), n, ctypes.byref(view), s, 1)
    assert rc == -1 and b"aligned" in L.ep_last_error()
    # a device buffer shorter than the blob
    assert _noalloc(ep, comp, dev_blob, out, nbytes=n - 16) == -1
    assert b"smaller" in L.ep_last_error()
    # host output is not accepted
    host = torch.empty(comp.shape, dtype=torch.bfloat16)
    hv = ep.tensor_view(host)
    rc = L.ep_decompress_noalloc(comp.handle, ctypes.c_void_p(dev_blob.data_ptr()), n, ctypes.byref(hv), s, 1)
    assert rc == -1
    # wrong shape
    bad = ep.EpTensor(out.data_ptr(), out.device.index, 1, 255, 256, 256)
    rc = L.ep_decompress_noalloc(comp.handle, ctypes.c_void_p(dev_blob.data_ptr()), n, ctypes.byref(bad), s, 1)
    assert rc == -3
