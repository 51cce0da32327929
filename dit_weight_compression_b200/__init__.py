"""B200-native lattice-rANS weight codec (EntroPack-style): Python binding.

A thin ctypes layer over ``libentropack.so`` (declared in ``include/entropack.h``).  It only
marshals arguments: compression runs in the library's host encoder, and decompression is one
fused CUDA kernel on the caller's stream.  PyTorch supplies device memory and streams.

The call names follow the interface the method's documentation describes ("EntroPack lattice
compression", section "Usage"): a config object carrying the target rate, ``compress`` returning
an object with ``actual_bpp``, and ``decompress`` restoring shape and dtype.  For example::

    import dit_weight_compression_b200 as ep
    blob = ep.compress(w, ep.LatticeRANSConfig(4.0))   # w: 2-D bf16/fp16/fp8_e4m3fn/fp32/int8
    w_hat = ep.decompress(blob)                        # on the current GPU, same shape and dtype
    print(blob.actual_bpp)                             # stored bits per element, metadata included
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libentropack.so")

BF16, FP16, FP8_E4M3, F32, INT8 = 1, 2, 3, 4, 5
_TORCH_TO_EP = {torch.bfloat16: BF16, torch.float16: FP16, torch.float8_e4m3fn: FP8_E4M3,
                torch.float32: F32, torch.int8: INT8}
_EP_TO_TORCH = {v: k for k, v in _TORCH_TO_EP.items()}

ERRORS = {-1: "EP_ERR_ARG", -2: "EP_ERR_DTYPE", -3: "EP_ERR_SHAPE", -4: "EP_ERR_RANGE",
          -5: "EP_ERR_CORRUPT", -6: "EP_ERR_CUDA", -7: "EP_ERR_OOM"}

# C-ABI entry points declared in include/entropack.h, with their ctypes signatures.
_P, _I, _I64, _D, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double, ctypes.c_size_t


class EpTensor(ctypes.Structure):
    _fields_ = [("data", _P), ("device", _I), ("dtype", _I), ("rows", _I64), ("cols", _I64),
                ("row_stride", _I64)]


class EpOptions(ctypes.Structure):
    _fields_ = [("steps_per_tile", _I), ("num_threads", _I), ("scale", _D), ("rd_refine", _I),
                ("host_encoder", _I), ("prob_bits", _I)]


class EpBlobInfo(ctypes.Structure):
    _fields_ = [("rows", _I64), ("cols", _I64), ("dtype", _I), ("steps_per_tile", _I),
                ("n_tiles", _I64), ("n_vectors", _I64), ("scale", _D), ("bytes", ctypes.c_uint64),
                ("prob_bits", _I)]


SIGNATURES = {
    "ep_compress": (_I, [ctypes.POINTER(EpTensor), _D, ctypes.POINTER(_P)]),
    "ep_compress_ex": (_I, [ctypes.POINTER(EpTensor), _D, ctypes.POINTER(EpOptions), ctypes.POINTER(_P)]),
    "ep_decompress": (_I, [_P, ctypes.POINTER(EpTensor), _P]),
    "ep_decompress_group": (_I, [ctypes.POINTER(_P), ctypes.POINTER(EpTensor), _I, _P]),
    "ep_actual_bpp": (_D, [_P]),
    "ep_get_info": (_I, [_P, ctypes.POINTER(EpBlobInfo)]),
    "ep_blob_to_bytes": (_I, [_P, ctypes.POINTER(_P), ctypes.POINTER(_SZ)]),
    "ep_blob_from_bytes": (_I, [_P, _SZ, ctypes.POINTER(_P)]),
    "ep_blob_prepare": (_I, [_P, _I, _P]),
    "ep_decode_status": (_I, [_P, _P]),
    "ep_decode_shape": (_I, [_P, ctypes.POINTER(_I), ctypes.POINTER(_I)]),
    "ep_decode_fields": (_I, [_P, _P, _P]),
    "ep_decompress_noalloc": (_I, [_P, _P, _SZ, ctypes.POINTER(EpTensor), _P, _I]),
    "ep_decode_wait_probe": (_I, [_P, ctypes.c_uint32, _P]),
    "ep_decompress_fp8_rowscaled": (_I, [_P, ctypes.POINTER(EpTensor), _P, _P]),
    "ep_blob_free": (None, [_P]),
    "ep_last_error": (ctypes.c_char_p, []),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C library.  Raises if it has not been built (no fallback of any kind)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m dit_weight_compression_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


class EPError(RuntimeError):
    def __init__(self, code: int, where: str):
        msg = lib().ep_last_error().decode(errors="replace")
        super().__init__(f"{where}: {ERRORS.get(code, code)}: {msg}")
        self.code = code


def _check(rc: int, where: str) -> None:
    if rc != 0:
        raise EPError(rc, where)


def _stream_handle(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def tensor_view(t: torch.Tensor) -> EpTensor:
    """The C view of a 2-D tensor with unit column stride."""
    if t.dim() != 2:
        raise ValueError("expected a 2-D tensor")
    if t.dtype not in _TORCH_TO_EP:
        raise TypeError(f"unsupported dtype {t.dtype}")
    if t.stride(1) != 1 and t.shape[1] > 1:
        raise ValueError("columns must be contiguous (stride 1)")
    dev = t.device.index if t.is_cuda else -1
    if t.is_cuda and dev is None:
        dev = torch.cuda.current_device()
    stride = t.stride(0) if t.shape[0] > 1 else t.shape[1]
    return EpTensor(t.data_ptr(), dev, _TORCH_TO_EP[t.dtype], t.shape[0], t.shape[1], max(stride, t.shape[1]))


@dataclass(frozen=True)
class LatticeRANSConfig:
    """Target storage rate in bits per element: finite, in [0.001, 11], non-integer allowed
    ("EntroPack lattice compression", opening paragraph)."""
    target_bpp: float
    steps_per_tile: int = 0     # rANS steps per tile (tile = 32 x S vectors); 0 = default rule
    num_threads: int = 0        # host encoder threads; 0 = all
    rd_refine: bool = False     # per-row rate-distortion refinement (slower encode; off by default)
    host_encoder: bool = False  # encode CUDA tensors on the host instead of on their GPU
    prob_bits: int = 12         # frequency totals 2^prob_bits: 12 (the format's choice) or 10 (faster decode)

    def __post_init__(self):
        t = float(self.target_bpp)
        if not (t == t and 0.001 <= t <= 11.0):
            raise ValueError("target_bpp must be finite and in [0.001, 11]")
        if self.prob_bits not in (10, 12):
            raise ValueError("prob_bits must be 12 or 10")


class CompressedTensor:
    """A compressed 2-D tensor (the library-owned blob)."""

    def __init__(self, handle: int):
        self._h = ctypes.c_void_p(handle)
        info = EpBlobInfo()
        _check(lib().ep_get_info(self._h, ctypes.byref(info)), "ep_get_info")
        self.info = info
        self.shape = (info.rows, info.cols)
        self.dtype = _EP_TO_TORCH[info.dtype]

    @property
    def handle(self) -> ctypes.c_void_p:
        return self._h

    @property
    def actual_bpp(self) -> float:
        return lib().ep_actual_bpp(self._h)

    @property
    def nbytes(self) -> int:
        return int(self.info.bytes)

    def to_bytes(self) -> bytes:
        p, n = ctypes.c_void_p(), ctypes.c_size_t()
        _check(lib().ep_blob_to_bytes(self._h, ctypes.byref(p), ctypes.byref(n)), "ep_blob_to_bytes")
        return ctypes.string_at(p, n.value)

    @classmethod
    def from_bytes(cls, data: bytes) -> "CompressedTensor":
        h = ctypes.c_void_p()
        buf = ctypes.create_string_buffer(bytes(data), len(data))
        _check(lib().ep_blob_from_bytes(buf, len(data), ctypes.byref(h)), "ep_blob_from_bytes")
        return cls(h.value)

    def prepare(self, device: int | None = None, stream=None) -> None:
        """Copy the blob to `device` now (keeps allocation out of timed or captured regions)."""
        dev = torch.cuda.current_device() if device is None else device
        with torch.cuda.device(dev):
            _check(lib().ep_blob_prepare(self._h, dev, _stream_handle(stream)), "ep_blob_prepare")

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value and _lib is not None:
            _lib.ep_blob_free(h)
            self._h = ctypes.c_void_p()


def compress(tensor: torch.Tensor, config, *, scale: float = 0.0) -> CompressedTensor:
    """Compress a 2-D tensor.  `config` is a LatticeRANSConfig or a target bpp."""
    cfg = config if isinstance(config, LatticeRANSConfig) else LatticeRANSConfig(float(config))
    t = tensor
    if t.dim() != 2:
        raise ValueError("expected a 2-D tensor")
    if t.stride(1) != 1 and t.shape[1] > 1:
        t = t.contiguous()
    view = tensor_view(t)
    opts = EpOptions(cfg.steps_per_tile, cfg.num_threads, float(scale), int(bool(cfg.rd_refine)),
                     int(bool(cfg.host_encoder)), int(cfg.prob_bits))
    h = ctypes.c_void_p()
    _check(lib().ep_compress_ex(ctypes.byref(view), cfg.target_bpp, ctypes.byref(opts), ctypes.byref(h)),
           "ep_compress")
    return CompressedTensor(h.value)


def decompress(compressed: CompressedTensor, config=None, *, out: torch.Tensor | None = None,
               dtype: torch.dtype | None = None, device=None, stream=None) -> torch.Tensor:
    """Decode to a tensor of the original shape (and dtype unless `dtype` or `out` say otherwise).
    A CUDA `out` (or the default) is written asynchronously by one kernel on `stream`; a CPU
    `out` runs the end-to-end path (upload, decode, download) and returns when it is done."""
    if out is None:
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        out = torch.empty(compressed.shape, dtype=dtype or compressed.dtype, device=dev)
    view = tensor_view(out)
    if out.is_cuda:
        with torch.cuda.device(out.device):
            _check(lib().ep_decompress(compressed.handle, ctypes.byref(view), _stream_handle(stream)),
                   "ep_decompress")
    else:
        _check(lib().ep_decompress(compressed.handle, ctypes.byref(view), _stream_handle(stream)),
               "ep_decompress")
    return out


def decompress_group(compressed: list, *, outs: list | None = None, dtype: torch.dtype | None = None,
                     device=None, stream=None) -> list:
    """Decode several blobs (e.g. one block's linear layers) with ep_decompress_group: one kernel
    launch per 28 blobs of one frequency-total width, results bit-identical to decompress().  Outputs are CUDA tensors of one
    dtype (the first blob's unless `dtype` or `outs` say otherwise), written asynchronously."""
    n = len(compressed)
    if outs is None:
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        dt = dtype or (compressed[0].dtype if n else torch.bfloat16)
        outs = [torch.empty(c.shape, dtype=dt, device=dev) for c in compressed]
    if len(outs) != n:
        raise ValueError("decompress_group: one output per blob")
    if n == 0:
        return outs
    handles = (_P * n)(*[c.handle.value for c in compressed])
    views = (EpTensor * n)(*[tensor_view(o) for o in outs])
    if outs[0].is_cuda:
        with torch.cuda.device(outs[0].device):
            _check(lib().ep_decompress_group(handles, views, n, _stream_handle(stream)), "ep_decompress_group")
    else:  # rejected by the library (device outputs only)
        _check(lib().ep_decompress_group(handles, views, n, _stream_handle(stream)), "ep_decompress_group")
    return outs


def decompress_fp8_rowscaled(compressed: CompressedTensor, *, out: torch.Tensor | None = None,
                             row_scale: torch.Tensor | None = None, device=None, stream=None):
    """The FP8 container with a per-row scale: returns (payload, row_scale), an E4M3 tensor of the
    blob's shape normalised per row to +-448 and a float32 vector with one scale per row, such
    that row_scale[:, None] * payload.float() restores the weights.  One kernel on `stream`."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if out is None:
        out = torch.empty(compressed.shape, dtype=torch.float8_e4m3fn, device=dev)
    if row_scale is None:
        row_scale = torch.empty(compressed.shape[0], dtype=torch.float32, device=out.device)
    if row_scale.dtype != torch.float32 or row_scale.numel() != compressed.shape[0] or not row_scale.is_contiguous():
        raise ValueError("row_scale must be a contiguous float32 vector with one entry per row")
    view = tensor_view(out)

    def call():
        _check(lib().ep_decompress_fp8_rowscaled(compressed.handle, ctypes.byref(view),
                                                 ctypes.c_void_p(row_scale.data_ptr()), _stream_handle(stream)),
               "ep_decompress_fp8_rowscaled")

    if out.is_cuda:
        with torch.cuda.device(out.device):
            call()
    else:  # rejected by the library (device outputs only)
        call()
    return out, row_scale


def decode_status(compressed: CompressedTensor, stream=None) -> None:
    """Raise EPError if any decode of this blob on the current device found corrupt tiles."""
    _check(lib().ep_decode_status(compressed.handle, _stream_handle(stream)), "ep_decode_status")


def decode_shape(compressed: CompressedTensor) -> tuple[int, int]:
    """(table layout, CTA width in warps) of decompress() for this blob on the current device."""
    lay, warps = _I(0), _I(0)
    _check(lib().ep_decode_shape(compressed.handle, ctypes.byref(lay), ctypes.byref(warps)), "ep_decode_shape")
    return lay.value, warps.value


def decode_fields(compressed: CompressedTensor, stream=None) -> torch.Tensor:
    """(n_vectors, 9) int16 on the current device: coset bit, then fields f1..f8."""
    out = torch.empty((compressed.info.n_vectors, 9), dtype=torch.int16, device="cuda")
    _check(lib().ep_decode_fields(compressed.handle, ctypes.c_void_p(out.data_ptr()), _stream_handle(stream)),
           "ep_decode_fields")
    return out


__all__ = ["LatticeRANSConfig", "CompressedTensor", "compress", "decompress", "decompress_group",
           "decompress_fp8_rowscaled", "decode_status",
           "decode_fields", "EPError", "lib", "BF16", "FP16", "FP8_E4M3", "F32", "INT8"]
