"""CPU oracle for the FP6 (e3m2) x FP16 weight-only linear layer.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package.  The CUDA
library and its Python binding never import it, and it shares no code with
them.  The arithmetic lives in ``fp6_oracle.c`` (plain C, binary64); this
module only builds that file with gcc and marshals numpy arrays through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp6_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED_SHAPE = 2
ERR_NONFINITE = 4
ERR_SCALE_RANGE = 5


def build(force: bool = False) -> str:
    """Compile fp6_oracle.c into liboracle.so (gcc, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
               "-ffp-contract=off", "-pthread", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            lib.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
            lib.oracle_f16_to_f64.restype = ctypes.c_double
            lib.oracle_f64_to_f16_rne.argtypes = [ctypes.c_double]
            lib.oracle_f64_to_f16_rne.restype = ctypes.c_uint16
            lib.oracle_round_e3m2.argtypes = [ctypes.c_double]
            lib.oracle_round_e3m2.restype = ctypes.c_uint8
            lib.oracle_decode_table.argtypes = [P]
            lib.oracle_decode_table.restype = None
            lib.oracle_quantize.argtypes = [P, I64, I64, P, P]
            lib.oracle_prepack.argtypes = [P, I64, I64, P]
            lib.oracle_unpack.argtypes = [P, I64, I64, P]
            lib.oracle_dequant.argtypes = [P, P, I64, I64, P]
            lib.oracle_linear.argtypes = [P, P, P, I64, I64, I64, P, ctypes.c_int]
            for f in ("oracle_quantize", "oracle_prepack", "oracle_unpack",
                      "oracle_dequant", "oracle_linear"):
                getattr(lib, f).restype = ctypes.c_int
            I = ctypes.c_int
            lib.oracle_fpx_codes.argtypes = [I]
            lib.oracle_fpx_decode_table.argtypes = [I, P]
            lib.oracle_fpx_round.argtypes = [I, ctypes.c_double]
            lib.oracle_fpx_quantize.argtypes = [I, P, I64, I64, P, P]
            lib.oracle_fpx_packed_bytes.argtypes = [I, I64, I64]
            lib.oracle_fpx_packed_bytes.restype = I64
            lib.oracle_fpx_prepack.argtypes = [I, P, I64, I64, P]
            lib.oracle_fpx_unpack.argtypes = [I, P, I64, I64, P]
            lib.oracle_fpx_dequant.argtypes = [I, P, P, I64, I64, P]
            lib.oracle_fpx_linear.argtypes = [I, P, P, P, I64, I64, I64, P]
            for f in ("oracle_fpx_codes", "oracle_fpx_decode_table", "oracle_fpx_round", "oracle_fpx_quantize",
                      "oracle_fpx_prepack", "oracle_fpx_unpack", "oracle_fpx_dequant", "oracle_fpx_linear"):
                getattr(lib, f).restype = ctypes.c_int
            lib.oracle_s24_quantize.argtypes = [P, I64, I64, P, P, P]
            lib.oracle_s24_packed_bytes.argtypes = [I64, I64]
            lib.oracle_s24_packed_bytes.restype = I64
            lib.oracle_s24_prepack.argtypes = [P, P, I64, I64, P]
            lib.oracle_s24_unpack.argtypes = [P, I64, I64, P, P]
            lib.oracle_s24_dequant.argtypes = [P, P, I64, I64, P]
            lib.oracle_s24_linear.argtypes = [P, P, P, P, I64, I64, I64, P]
            for f in ("oracle_s24_quantize", "oracle_s24_prepack", "oracle_s24_unpack", "oracle_s24_dequant",
                      "oracle_s24_linear"):
                getattr(lib, f).restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


class OracleError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: oracle status {status}")
        self.status = status


def decode_table() -> np.ndarray:
    """Values of the 64 e3m2 codes (binary64)."""
    out = np.zeros(64, dtype=np.float64)
    _load().oracle_decode_table(_ptr(out))
    return out


def f16_to_f64(bits: int) -> float:
    return _load().oracle_f16_to_f64(int(bits))


def f64_to_f16(v: float) -> int:
    return int(_load().oracle_f64_to_f16_rne(float(v)))


def f64_to_f16_array(v: np.ndarray) -> np.ndarray:
    lib = _load()
    flat = np.asarray(v, dtype=np.float64).ravel()
    return np.array([lib.oracle_f64_to_f16_rne(float(a)) for a in flat], dtype=np.uint16).reshape(np.shape(v))


def round_e3m2(v: float) -> int:
    return int(_load().oracle_round_e3m2(float(v)))


def quantize(W: np.ndarray):
    """W float32 [N,K] -> (codes uint8 [N,K], scales fp16 bits uint16 [N])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    codes = np.zeros((N, K), dtype=np.uint8)
    scales = np.zeros(N, dtype=np.uint16)
    st = _load().oracle_quantize(_ptr(W), N, K, _ptr(codes), _ptr(scales))
    if st != OK:
        raise OracleError(st, "quantize")
    return codes, scales


def prepack(codes: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    N, K = codes.shape
    out = np.zeros(N * K * 3 // 4, dtype=np.uint8)
    st = _load().oracle_prepack(_ptr(codes), N, K, _ptr(out))
    if st != OK:
        raise OracleError(st, "prepack")
    return out


def unpack(packed: np.ndarray, N: int, K: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    codes = np.zeros((N, K), dtype=np.uint8)
    st = _load().oracle_unpack(_ptr(packed), N, K, _ptr(codes))
    if st != OK:
        raise OracleError(st, "unpack")
    return codes


def dequant(packed: np.ndarray, scales, N: int, K: int) -> np.ndarray:
    """-> fp16 bit patterns uint16 [N,K]."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    out = np.zeros((N, K), dtype=np.uint16)
    sp = None
    if scales is not None:
        scales = np.ascontiguousarray(scales, dtype=np.uint16)
        sp = _ptr(scales)
    st = _load().oracle_dequant(_ptr(packed), sp, N, K, _ptr(out))
    if st != OK:
        raise OracleError(st, "dequant")
    return out


def linear(x16: np.ndarray, codes: np.ndarray, scales: np.ndarray, nthreads: int = 1) -> np.ndarray:
    """x16: fp16 bits uint16 [M,K]; codes uint8 [N,K]; scales uint16 [N] -> y fp16 bits [M,N]."""
    x16 = np.ascontiguousarray(x16, dtype=np.uint16)
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    M, K = x16.shape
    N, K2 = codes.shape
    assert K == K2 and scales.shape == (N,)
    y = np.zeros((M, N), dtype=np.uint16)
    st = _load().oracle_linear(_ptr(x16), _ptr(codes), _ptr(scales), M, N, K, _ptr(y), int(nthreads))
    if st != OK:
        raise OracleError(st, "linear")
    return y


# ---- other FPx formats (0 = FP6 e3m2, 1 = FP6 e2m3, 2 = FP4 e2m1, 3 = FP5 e2m2) ----

E3M2, E2M3, E2M1, E2M2 = 0, 1, 2, 3


def fpx_codes(fmt: int) -> int:
    return int(_load().oracle_fpx_codes(int(fmt)))


def fpx_decode_table(fmt: int) -> np.ndarray:
    out = np.zeros(fpx_codes(fmt), dtype=np.float64)
    st = _load().oracle_fpx_decode_table(int(fmt), _ptr(out))
    if st != OK:
        raise OracleError(st, "fpx_decode_table")
    return out


def fpx_round(fmt: int, v: float) -> int:
    return int(_load().oracle_fpx_round(int(fmt), float(v)))


def fpx_quantize(fmt: int, W: np.ndarray):
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    codes = np.zeros((N, K), dtype=np.uint8)
    scales = np.zeros(N, dtype=np.uint16)
    st = _load().oracle_fpx_quantize(int(fmt), _ptr(W), N, K, _ptr(codes), _ptr(scales))
    if st != OK:
        raise OracleError(st, "fpx_quantize")
    return codes, scales


def fpx_packed_bytes(fmt: int, N: int, K: int) -> int:
    return int(_load().oracle_fpx_packed_bytes(int(fmt), N, K))


def fpx_prepack(fmt: int, codes: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    N, K = codes.shape
    out = np.zeros(fpx_packed_bytes(fmt, N, K), dtype=np.uint8)
    st = _load().oracle_fpx_prepack(int(fmt), _ptr(codes), N, K, _ptr(out))
    if st != OK:
        raise OracleError(st, "fpx_prepack")
    return out


def fpx_unpack(fmt: int, packed: np.ndarray, N: int, K: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    codes = np.zeros((N, K), dtype=np.uint8)
    st = _load().oracle_fpx_unpack(int(fmt), _ptr(packed), N, K, _ptr(codes))
    if st != OK:
        raise OracleError(st, "fpx_unpack")
    return codes


def fpx_dequant(fmt: int, packed: np.ndarray, scales, N: int, K: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    out = np.zeros((N, K), dtype=np.uint16)
    sp = None
    if scales is not None:
        scales = np.ascontiguousarray(scales, dtype=np.uint16)
        sp = _ptr(scales)
    st = _load().oracle_fpx_dequant(int(fmt), _ptr(packed), sp, N, K, _ptr(out))
    if st != OK:
        raise OracleError(st, "fpx_dequant")
    return out


def fpx_linear(fmt: int, x16: np.ndarray, codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    x16 = np.ascontiguousarray(x16, dtype=np.uint16)
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    M, K = x16.shape
    N, K2 = codes.shape
    assert K == K2 and scales.shape == (N,)
    y = np.zeros((M, N), dtype=np.uint16)
    st = _load().oracle_fpx_linear(int(fmt), _ptr(x16), _ptr(codes), _ptr(scales), M, N, K, _ptr(y))
    if st != OK:
        raise OracleError(st, "fpx_linear")
    return y


# ---- 2:4 sparse INT4 (Sparse-Marlin): kept codes, their positions, row scales ----


def s24_quantize(W: np.ndarray):
    """W [N,K] fp32 -> (q [N,K/2] int8, pos [N,K/2] uint8, scales [N] fp16 bits)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    q = np.zeros((N, K // 2), dtype=np.int8)
    pos = np.zeros((N, K // 2), dtype=np.uint8)
    scales = np.zeros(N, dtype=np.uint16)
    st = _load().oracle_s24_quantize(_ptr(W), N, K, _ptr(q), _ptr(pos), _ptr(scales))
    if st != OK:
        raise OracleError(st, "s24_quantize")
    return q, pos, scales


def s24_packed_bytes(N: int, K: int) -> int:
    return int(_load().oracle_s24_packed_bytes(N, K))


def s24_prepack(q: np.ndarray, pos: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.int8)
    pos = np.ascontiguousarray(pos, dtype=np.uint8)
    N, K2 = q.shape
    out = np.zeros(s24_packed_bytes(N, 2 * K2), dtype=np.uint8)
    st = _load().oracle_s24_prepack(_ptr(q), _ptr(pos), N, 2 * K2, _ptr(out))
    if st != OK:
        raise OracleError(st, "s24_prepack")
    return out


def s24_unpack(packed: np.ndarray, N: int, K: int):
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    q = np.zeros((N, K // 2), dtype=np.int8)
    pos = np.zeros((N, K // 2), dtype=np.uint8)
    st = _load().oracle_s24_unpack(_ptr(packed), N, K, _ptr(q), _ptr(pos))
    if st != OK:
        raise OracleError(st, "s24_unpack")
    return q, pos


def s24_dequant(packed: np.ndarray, scales, N: int, K: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    out = np.zeros((N, K), dtype=np.uint16)
    sp = None
    if scales is not None:
        scales = np.ascontiguousarray(scales, dtype=np.uint16)
        sp = _ptr(scales)
    st = _load().oracle_s24_dequant(_ptr(packed), sp, N, K, _ptr(out))
    if st != OK:
        raise OracleError(st, "s24_dequant")
    return out


def s24_linear(x16: np.ndarray, q: np.ndarray, pos: np.ndarray, scales: np.ndarray) -> np.ndarray:
    x16 = np.ascontiguousarray(x16, dtype=np.uint16)
    q = np.ascontiguousarray(q, dtype=np.int8)
    pos = np.ascontiguousarray(pos, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    M, K = x16.shape
    N = q.shape[0]
    assert q.shape == (N, K // 2) and pos.shape == q.shape and scales.shape == (N,)
    y = np.zeros((M, N), dtype=np.uint16)
    st = _load().oracle_s24_linear(_ptr(x16), _ptr(q), _ptr(pos), _ptr(scales), M, N, K, _ptr(y))
    if st != OK:
        raise OracleError(st, "s24_linear")
    return y
