"""FP6 (e3m2) x FP16 weight-only linear layer for NVIDIA B200 (sm_100a).

Thin PyTorch-facing wrapper over libfp6.so (include/fp6.h).  PyTorch provides
device memory and the current stream; every step of the computation runs in
the library's CUDA kernels.

    import weight_only_quantized_fp6_b200 as fp6
    layer = fp6.FP6Linear.from_float(W)        # W: [N,K] fp32 on cuda
    y = layer(x)                               # x: [M,K] fp16 on cuda -> [M,N] fp16

Every function takes an optional `fmt`: None (the default) is FP6 e3m2 through
the fp6_* entry points; E3M2, E2M3 (FP6 with two exponent bits), E2M1 (FP4)
or E2M2 (FP5) select the fpx_* entry points with that format, and S24 the
2:4-sparse INT4 weights of the s24_* entry points (quantized by
s24_quantize, which also returns the kept positions).
"""
from __future__ import annotations

import ctypes
import threading

from . import _lib

__all__ = ["quantize", "prepack", "dequant", "linear", "linear_plan", "workspace_bytes",
           "packed_bytes", "device_status", "FP6Linear", "FP6Error", "Workspace",
           "s24_quantize", "s24_prepack", "packed_header", "check_packed_header",
           "E3M2", "E2M3", "E2M1", "E2M2", "S24"]

FP6Error = _lib.FP6Error

# fpx_format values (include/fp6.h); S24 selects the s24_* entry points
E3M2, E2M3, E2M1, E2M2 = 0, 1, 2, 3
S24 = 4


def _check_fmt(fmt):
    if fmt is not None and fmt not in (E3M2, E2M3, E2M1, E2M2, S24):
        raise ValueError(f"unknown format {fmt!r}")


def _torch():
    import torch
    return torch


def _stream(t):
    return ctypes.c_void_p(_torch().cuda.current_stream(t.device).cuda_stream)


def _need_cuda(name, t, dtype, dim=None):
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if dim is not None and t.dim() != dim:
        raise ValueError(f"{name} must have {dim} dimensions")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


# Sizes the library reports, cached per shape: a layer called in a decode loop
# asks for the same few sizes every time, and each query is a foreign call.
_packed_bytes_cache = {}
_workspace_cache = {}


def packed_bytes(N: int, K: int, fmt=None) -> int:
    key = (N, K, fmt)
    v = _packed_bytes_cache.get(key)
    if v is None:
        _check_fmt(fmt)
        if fmt is None:
            v = int(_lib.load().fp6_packed_bytes(N, K))
        elif fmt == S24:
            v = int(_lib.load().s24_packed_bytes(N, K))
        else:
            v = int(_lib.load().fpx_packed_bytes(fmt, N, K))
        _packed_bytes_cache[key] = v
    return v


def quantize(W, fmt=None):
    """W [N,K] fp32 (cuda) -> (codes [N,K] uint8, scales [N] fp16).  Synchronizes."""
    torch = _torch()
    _check_fmt(fmt)
    if fmt == S24:
        raise ValueError("2:4 sparse weights are quantized by s24_quantize")
    _need_cuda("W", W, torch.float32, 2)
    N, K = W.shape
    codes = torch.empty((N, K), dtype=torch.uint8, device=W.device)
    scales = torch.empty((N,), dtype=torch.float16, device=W.device)
    lib = _lib.load()
    if fmt is None:
        st = lib.fp6_quantize(W.data_ptr(), N, K, codes.data_ptr(), scales.data_ptr(), _stream(W))
    else:
        st = lib.fpx_quantize(fmt, W.data_ptr(), N, K, codes.data_ptr(), scales.data_ptr(), _stream(W))
    _lib.check(st, "fp6_quantize" if fmt is None else "fpx_quantize")
    return codes, scales


def prepack(codes, fmt=None):
    """codes [N,K] uint8 (cuda) -> packed uint8 buffer (3*N*K/4 bytes; N*K/2 for E2M1, 5*N*K/8 for E2M2)."""
    torch = _torch()
    if fmt == S24:
        raise ValueError("2:4 sparse weights are packed by s24_prepack")
    _need_cuda("codes", codes, torch.uint8, 2)
    N, K = codes.shape
    nbytes = packed_bytes(N, K, fmt)
    if nbytes == 0 and N * K > 0:
        raise FP6Error(2, "fp6_prepack")
    packed = torch.empty((nbytes,), dtype=torch.uint8, device=codes.device)
    lib = _lib.load()
    if fmt is None:
        st = lib.fp6_prepack(codes.data_ptr(), N, K, packed.data_ptr(), nbytes, _stream(codes))
    else:
        st = lib.fpx_prepack(fmt, codes.data_ptr(), N, K, packed.data_ptr(), nbytes, _stream(codes))
    _lib.check(st, "fp6_prepack" if fmt is None else "fpx_prepack")
    return packed


def dequant(packed, scales, N: int, K: int, fmt=None, out=None):
    """packed -> W16 [N,K] fp16 (into `out` when given); scales None gives the
    unscaled code values."""
    torch = _torch()
    _check_fmt(fmt)
    _need_cuda("packed", packed, torch.uint8, 1)
    if scales is not None:
        _need_cuda("scales", scales, torch.float16, 1)
    if out is None:
        out = torch.empty((N, K), dtype=torch.float16, device=packed.device)
    else:
        _need_cuda("out", out, torch.float16, 2)
        if tuple(out.shape) != (N, K):
            raise ValueError(f"out must be [{N}, {K}]")
    sp = scales.data_ptr() if scales is not None else None
    lib = _lib.load()
    if fmt is None:
        st = lib.fp6_dequant(packed.data_ptr(), sp, N, K, out.data_ptr(), _stream(packed))
    elif fmt == S24:
        st = lib.s24_dequant(packed.data_ptr(), sp, N, K, out.data_ptr(), _stream(packed))
    else:
        st = lib.fpx_dequant(fmt, packed.data_ptr(), sp, N, K, out.data_ptr(), _stream(packed))
    _lib.check(st, "fp6_dequant" if fmt is None else "fpx_dequant")
    return out


def s24_quantize(W):
    """W [N,K] fp32 (cuda, K % 4 == 0) -> (q [N,K/2] int8, pos [N,K/2] uint8,
    scales [N] fp16): in each group of four the two largest |w| kept, their
    codes round-half-even(w/scale) in [-8, 7] and positions.  Synchronizes."""
    torch = _torch()
    _need_cuda("W", W, torch.float32, 2)
    N, K = W.shape
    q = torch.empty((N, K // 2), dtype=torch.int8, device=W.device)
    pos = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
    scales = torch.empty((N,), dtype=torch.float16, device=W.device)
    st = _lib.load().s24_quantize(W.data_ptr(), N, K, q.data_ptr(), pos.data_ptr(), scales.data_ptr(), _stream(W))
    _lib.check(st, "s24_quantize")
    return q, pos, scales


def s24_prepack(q, pos):
    """(q, pos) [N,K/2] -> packed uint8 buffer of 3*N*K/8 bytes."""
    torch = _torch()
    _need_cuda("q", q, torch.int8, 2)
    _need_cuda("pos", pos, torch.uint8, 2)
    N, K2 = q.shape
    K = 2 * K2
    nbytes = packed_bytes(N, K, S24)
    if nbytes == 0 and N * K > 0:
        raise FP6Error(2, "s24_prepack")
    packed = torch.empty((nbytes,), dtype=torch.uint8, device=q.device)
    st = _lib.load().s24_prepack(q.data_ptr(), pos.data_ptr(), N, K, packed.data_ptr(), nbytes, _stream(q))
    _lib.check(st, "s24_prepack")
    return packed


def workspace_bytes(M: int, N: int, K: int) -> int:
    """Workspace fp6_linear needs on the current device (it depends on the
    device's SM count, so the cache is keyed by device)."""
    key = (_torch().cuda.current_device(), M, N, K)
    v = _workspace_cache.get(key)
    if v is None:
        v = int(_lib.load().fp6_linear_workspace_bytes(M, N, K))
        _workspace_cache[key] = v
    return v


def linear_plan(M: int, N: int, K: int) -> dict:
    out = (ctypes.c_int64 * 5)()
    _lib.check(_lib.load().fp6_linear_plan(M, N, K, out), "fp6_linear_plan")
    return {"ncol": out[0], "stages": out[1], "grid": out[2], "tiles": out[3], "iters": out[4]}


class Workspace:
    """A zero-initialised device buffer reused across fp6_linear calls on one
    device and stream (the kernels leave its counters zero after each call)."""

    def __init__(self, device=None):
        self.device = device
        self.buf = None

    def get(self, nbytes: int):
        torch = _torch()
        if nbytes == 0:
            return None
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.zeros((max(nbytes, 1 << 20),), dtype=torch.uint8, device=self.device)
        return self.buf


_ws_lock = threading.Lock()
_default_ws = {}


def _default_workspace(device):
    key = (device.type, device.index, _torch().cuda.current_stream(device).cuda_stream)
    with _ws_lock:
        if key not in _default_ws:
            _default_ws[key] = Workspace(device)
        return _default_ws[key]


def linear(x, packed, scales, N: int, K: int, out=None, workspace: Workspace | None = None, fmt=None):
    """y[M,N] = x[M,K] . (scales (.) decode(W))^T in fp16 (fp32 accumulation)."""
    torch = _torch()
    _check_fmt(fmt)
    _need_cuda("x", x, torch.float16, 2)
    _need_cuda("packed", packed, torch.uint8, 1)
    _need_cuda("scales", scales, torch.float16, 1)
    M, K2 = x.shape
    if K2 != K or scales.shape[0] != N:
        raise ValueError("shape mismatch between x, scales and (N, K)")
    if N > 0 and K > 0 and packed.numel() < packed_bytes(N, K, fmt):
        raise ValueError(f"packed holds {packed.numel()} bytes; an {N} x {K} weight needs "
                         f"{packed_bytes(N, K, fmt)}")
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=x.device)
    else:
        _need_cuda("out", out, torch.float16, 2)
    need = workspace_bytes(M, N, K)
    ws = (workspace or _default_workspace(x.device)).get(need)
    args = (x.data_ptr(), packed.data_ptr(), scales.data_ptr(), M, N, K, out.data_ptr(),
            ws.data_ptr() if ws is not None else None, ws.numel() if ws is not None else 0, _stream(x))
    lib = _lib.load()
    if fmt is None:
        _lib.check(lib.fp6_linear(*args), "fp6_linear")
    elif fmt == S24:
        _lib.check(lib.s24_linear(*args), "s24_linear")
    else:
        _lib.check(lib.fpx_linear(fmt, *args), "fpx_linear")
    return out


def device_status(device=None) -> int:
    """Reads and clears the kernels' device error word (0 = OK, 9 = a bounded wait timed out)."""
    torch = _torch()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    return int(_lib.load().fp6_get_device_status(ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)))


HEADER_BYTES = 64


def packed_header(N: int, K: int, fmt=None) -> bytes:
    """The 64-byte header of a stored N x K packed weight (include/fp6.h)."""
    _check_fmt(fmt)
    buf = ctypes.create_string_buffer(HEADER_BYTES)
    _lib.check(_lib.load().fp6_packed_header(E3M2 if fmt is None else fmt, N, K, buf), "fp6_packed_header")
    return buf.raw


def check_packed_header(header: bytes, N: int, K: int, fmt=None) -> None:
    """Raises FP6Error(FP6_ERR_LAYOUT_VERSION) unless `header` is what this
    library writes for an N x K weight in `fmt`."""
    _check_fmt(fmt)
    if len(header) < HEADER_BYTES:
        raise FP6Error(7, "fp6_packed_header_check")
    buf = ctypes.create_string_buffer(bytes(header[:HEADER_BYTES]), HEADER_BYTES)
    _lib.check(_lib.load().fp6_packed_header_check(buf, E3M2 if fmt is None else fmt, N, K),
               "fp6_packed_header_check")


class FP6Linear:
    """A linear layer whose weight is stored pre-packed (FP6 e3m2 unless `fmt`
    says otherwise) plus fp16 row scales."""

    def __init__(self, packed, scales, N: int, K: int, fmt=None):
        _check_fmt(fmt)
        self.packed, self.scales, self.N, self.K, self.fmt = packed, scales, N, K, fmt
        self.workspace = Workspace(packed.device)

    @classmethod
    def from_float(cls, W, fmt=None):
        if fmt == S24:
            q, pos, scales = s24_quantize(W)
            return cls(s24_prepack(q, pos), scales, W.shape[0], W.shape[1], fmt)
        codes, scales = quantize(W, fmt)
        return cls(prepack(codes, fmt), scales, W.shape[0], W.shape[1], fmt)

    def __call__(self, x, out=None):
        return linear(x, self.packed, self.scales, self.N, self.K, out=out, workspace=self.workspace,
                      fmt=self.fmt)

    def save(self, path) -> None:
        """Writes the layer as a stored blob: the 64-byte header, the fp16
        scales, the packed bytes."""
        torch = _torch()
        with open(path, "wb") as f:
            f.write(packed_header(self.N, self.K, self.fmt))
            f.write(self.scales.cpu().view(torch.int16).numpy().tobytes())
            f.write(self.packed.cpu().numpy().tobytes())

    @classmethod
    def load(cls, path, device="cuda"):
        """Reads a blob written by save(); raises FP6Error(FP6_ERR_LAYOUT_VERSION)
        when its header is not what this library writes for the shape and
        format it names (for example a blob packed under another layout)."""
        import struct
        import numpy as np
        torch = _torch()
        with open(path, "rb") as f:
            header = f.read(HEADER_BYTES)
            if len(header) < HEADER_BYTES or header[:4] != b"FP6W":
                raise FP6Error(7, "FP6Linear.load")
            fmt_code, = struct.unpack_from("<I", header, 8)
            N, K = struct.unpack_from("<qq", header, 16)
            fmt = None if fmt_code == E3M2 else int(fmt_code)
            if fmt not in (None, E2M3, E2M1, E2M2, S24):
                raise FP6Error(7, "FP6Linear.load")
            check_packed_header(header, N, K, fmt)
            scales = np.frombuffer(f.read(2 * N), dtype=np.int16)
            nbytes = packed_bytes(N, K, fmt)
            packed = np.frombuffer(f.read(nbytes), dtype=np.uint8)
            if scales.size != N or packed.size != nbytes:
                raise FP6Error(7, "FP6Linear.load")
        dev = torch.device(device)
        return cls(torch.from_numpy(packed.copy()).to(dev),
                   torch.from_numpy(scales.copy()).to(dev).view(torch.float16), N, K, fmt)
