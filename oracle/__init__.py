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
