"""ctypes binding of libfp6.so: argument marshalling only.

Every computation runs in the library's CUDA kernels.  Loading fails loudly if
the library has not been built; nothing here falls back to another
implementation.
"""
from __future__ import annotations

import ctypes
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libfp6.so")

STATUS = {
    0: "FP6_OK", 1: "FP6_ERR_INVALID_ARG", 2: "FP6_ERR_UNSUPPORTED_SHAPE", 3: "FP6_ERR_MISALIGNED",
    4: "FP6_ERR_NONFINITE", 5: "FP6_ERR_SCALE_RANGE", 6: "FP6_ERR_WORKSPACE", 7: "FP6_ERR_LAYOUT_VERSION",
    8: "FP6_ERR_CUDA",
    9: "FP6_ERR_TIMEOUT",
}

# name -> (restype, argtypes), mirroring include/fp6.h
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_ST = ctypes.c_int
SIGNATURES = {
    "fp6_status_string": (ctypes.c_char_p, [_ST]),
    "fp6_packed_bytes": (_SZ, [_I64, _I64]),
    "fp6_quantize": (_ST, [_P, _I64, _I64, _P, _P, _P]),
    "fp6_prepack": (_ST, [_P, _I64, _I64, _P, _SZ, _P]),
    "fp6_dequant": (_ST, [_P, _P, _I64, _I64, _P, _P]),
    "fp6_linear_workspace_bytes": (_SZ, [_I64, _I64, _I64]),
    "fp6_linear": (_ST, [_P, _P, _P, _I64, _I64, _I64, _P, _P, _SZ, _P]),
    "fp6_get_device_status": (_ST, [_P]),
    "fp6_linear_plan": (_ST, [_I64, _I64, _I64, ctypes.POINTER(_I64)]),
    "fp6_linear_plan_for_sms": (_ST, [_I64, _I64, _I64, ctypes.c_int, ctypes.POINTER(_I64)]),
    "fp6_linear_noalloc": (_ST, [_P, _P, _P, _I64, _I64, _I64, _P, _P]),
    "fp6_selftest_wait_timeout": (_ST, [_P]),
    "fpx_packed_bytes": (_SZ, [_ST, _I64, _I64]),
    "fpx_quantize": (_ST, [_ST, _P, _I64, _I64, _P, _P, _P]),
    "fpx_prepack": (_ST, [_ST, _P, _I64, _I64, _P, _SZ, _P]),
    "fpx_dequant": (_ST, [_ST, _P, _P, _I64, _I64, _P, _P]),
    "fpx_linear": (_ST, [_ST, _P, _P, _P, _I64, _I64, _I64, _P, _P, _SZ, _P]),
    "s24_packed_bytes": (_SZ, [_I64, _I64]),
    "s24_quantize": (_ST, [_P, _I64, _I64, _P, _P, _P, _P]),
    "s24_prepack": (_ST, [_P, _P, _I64, _I64, _P, _SZ, _P]),
    "s24_dequant": (_ST, [_P, _P, _I64, _I64, _P, _P]),
    "s24_linear": (_ST, [_P, _P, _P, _I64, _I64, _I64, _P, _P, _SZ, _P]),
    "fp6_packed_header": (_ST, [_ST, _I64, _I64, _P]),
    "fp6_packed_header_check": (_ST, [_P, _ST, _I64, _I64]),
}

_lock = threading.Lock()
_lib = None


class FP6Error(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what} failed: {STATUS.get(status, status)}")
        self.status = status


def load() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"libfp6.so not found at {LIB_PATH}; build it with "
                    "`python -m weight_only_quantized_fp6_b200.build` (needs nvcc, sm_100a)")
            lib = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                f = getattr(lib, name)
                f.restype = res
                f.argtypes = args
            _lib = lib
    return _lib


def check(status: int, what: str) -> None:
    if status != 0:
        raise FP6Error(status, what)
