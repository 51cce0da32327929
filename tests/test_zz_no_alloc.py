"""The allocation-free decode entry point, ep_decompress_noalloc, through the C ABI.

Some callers cannot let a library allocate GPU memory: an inference runtime that lays out all
device memory ahead of time in its own arena, or code running where an allocation is forbidden
or would synchronise the device.  For them ep_decompress_noalloc takes the blob's bytes already
in device memory (their allocation, not the library's) and keeps the decode kernel's status word
in a fixed array inside the library instead of allocating one.

This file checks that entry point against the ordinary ep_decompress on the same blob, bit for
bit (the tolerance the parity tests use), on two calls in a row, and that the two calls leave
the device's free memory unchanged.  It is named so that pytest collects it after every other
test file.
"""
import ctypes

import numpy as np
import pytest
import torch

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


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy()


def test_noalloc_matches_decompress_twice(ep):
    m = W.square(rows=1024, cols=2048)
    comp = ep.compress(W.bits_to_torch(m.bits, m.dtype), m.target_bpp)

    # reference: the ordinary entry point (it allocates its own device copy of the blob)
    ref = ep.decompress(comp)
    torch.cuda.synchronize()
    ep.decode_status(comp)

    # the caller owns the device copy of the bytes
    blob = comp.to_bytes()
    dev_blob = torch.frombuffer(bytearray(blob), dtype=torch.uint8).cuda()
    assert dev_blob.data_ptr() % 16 == 0
    stream = torch.cuda.current_stream()
    L = ep.lib()

    outs = [torch.full(comp.shape, float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    views = [ep.tensor_view(o) for o in outs]
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    for i in range(2):
        rc = L.ep_decompress_noalloc(comp.handle, ctypes.c_void_p(dev_blob.data_ptr()),
                                     ctypes.byref(views[i]), ctypes.c_void_p(stream.cuda_stream), 1)
        assert rc == 0, L.ep_last_error()
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    for o in outs:
        assert np.array_equal(_bits(o), _bits(ref))
    assert free_after == free_before


def test_noalloc_rejects_bad_arguments(ep):
    m = W.small()
    comp = ep.compress(W.bits_to_torch(m.bits, m.dtype), m.target_bpp)
    dev_blob = torch.frombuffer(bytearray(comp.to_bytes()), dtype=torch.uint8).cuda()
    out = torch.empty(comp.shape, dtype=torch.bfloat16, device="cuda")
    view = ep.tensor_view(out)
    L = ep.lib()
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # misaligned device bytes
    rc = L.ep_decompress_noalloc(comp.handle, ctypes.c_void_p(dev_blob.data_ptr() + 8), ctypes.byref(view), s, 1)
    assert rc == -1 and b"aligned" in L.ep_last_error()
    # host output is not accepted
    host = torch.empty(comp.shape, dtype=torch.bfloat16)
    hv = ep.tensor_view(host)
    rc = L.ep_decompress_noalloc(comp.handle, ctypes.c_void_p(dev_blob.data_ptr()), ctypes.byref(hv), s, 1)
    assert rc == -1
    # wrong shape
    bad = ep.EpTensor(out.data_ptr(), out.device.index, 1, 255, 256, 256)
    rc = L.ep_decompress_noalloc(comp.handle, ctypes.c_void_p(dev_blob.data_ptr()), ctypes.byref(bad), s, 1)
    assert rc == -3
