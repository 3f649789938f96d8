"""Pins for the oracle's FP6 quantizer (per-row fp16 scale, RNE e3m2 codes).

Reading of the layer's specification: s[n] = fp16_rne(fp32(max_k |W[n,k]| / 28)),
code = round-to-nearest-even of W/s onto the e3m2 grid, saturating at +-28,
sign kept.  The FP6-LLM abstract only says the weights are quantized to FP6.
"""
import ctypes
import os
import shutil
import subprocess
from fractions import Fraction

import numpy as np
import pytest

from tests.test_oracle_decode import closed_form

MAGS = [closed_form(c) for c in range(32)]


def brute_force_code(v: float) -> int:
    """argmin over the 32 e3m2 magnitudes of |v| - mag, ties to the even code;
    values beyond 28 saturate to 28; sign copied from v."""
    a = abs(Fraction(v))
    best, bestd = None, None
    for c, mag in enumerate(MAGS):
        d = abs(a - mag)
        if bestd is None or d < bestd or (d == bestd and c % 2 == 0):
            best, bestd = c, d
    sign = 0x20 if np.signbit(v) else 0
    return sign | best


def probe_values():
    rng = np.random.default_rng(7)
    mags = [float(m) for m in MAGS]
    mids = [(mags[i] + mags[i + 1]) / 2 for i in range(31)] + [30.0]
    vals = []
    for m in mids + mags:
        vals += [m, float(np.nextafter(m, 0)), float(np.nextafter(m, 100))]
    vals += list(rng.uniform(0, 40, 3000)) + list(rng.uniform(0, 0.3, 2000))
    vals += list(np.abs(rng.standard_normal(2000)) * 7)
    vals += [0.0, 1e-300, 28.0, 29.999, 30.0, 30.0001, 1e30]
    return vals + [-v for v in vals]


def test_round_e3m2_vs_brute_force(orc):
    for v in probe_values():
        assert orc.round_e3m2(v) == brute_force_code(v), v


def test_round_e3m2_error_bound(orc):
    """|v - decode(code)| <= half the spacing of v's binade (2^-5 below 0.25)."""
    for v in probe_values():
        a = abs(v)
        if a > 28:
            continue
        c = orc.round_e3m2(v)
        got = abs(MAGS[c & 0x1F])
        if a < 0.25:
            half = Fraction(1, 32)
        else:
            e = int(np.floor(np.log2(a)))
            half = Fraction(2) ** (e - 3)
        assert abs(Fraction(a) - got) <= half, v


@pytest.fixture(scope="module")
def cuda_fp6_cvt(tmp_path_factory):
    """CUDA's own host-side double->e3m2 conversion (cuda_fp6.h), called as a
    library routine for an independent second opinion."""
    hdr = "/usr/local/cuda/include/cuda_fp6.h"
    if not os.path.exists(hdr) or shutil.which("g++") is None:
        pytest.skip("cuda_fp6.h or g++ unavailable")
    d = tmp_path_factory.mktemp("fp6cvt")
    src = d / "cvt.cpp"
    src.write_text('#include <cuda_fp6.h>\n'
                   'extern "C" unsigned char cvt(double x){'
                   'return (unsigned char)__nv_cvt_double_to_fp6(x, __NV_E3M2, cudaRoundNearest);}\n')
    so = d / "cvt.so"
    subprocess.run(["g++", "-O1", "-shared", "-fPIC", "-I/usr/local/cuda/include",
                    str(src), "-o", str(so)], check=True)
    lib = ctypes.CDLL(str(so))
    lib.cvt.argtypes = [ctypes.c_double]
    lib.cvt.restype = ctypes.c_uint8
    return lib.cvt


def test_round_e3m2_vs_cuda_fp6_library(orc, cuda_fp6_cvt):
    for v in probe_values():
        assert orc.round_e3m2(v) == cuda_fp6_cvt(v), v


def test_scale_is_fp16_of_fp32_amax_over_28(orc):
    from weight_only_quantized_fp6_b200 import inputs
    W = inputs.weights(5, 64, 256)
    W[3, 17] = -0.75  # row whose max |w| is a negative weight
    codes, scales = orc.quantize(W)
    amax = np.abs(W).max(axis=1).astype(np.float32)
    ref = (amax / np.float32(28.0)).astype(np.float16).view(np.uint16)
    assert np.array_equal(scales, ref)


def test_quantize_codes_vs_brute_force(orc):
    from weight_only_quantized_fp6_b200 import inputs
    W = inputs.weights(11, 8, 512, outlier_p=0.01)
    codes, scales = orc.quantize(W)
    for n in range(8):
        s = float(np.array([scales[n]], dtype=np.uint16).view(np.float16)[0])
        for k in range(0, 512, 3):
            # exact quotient; brute force works on the rational w/s
            v = Fraction(float(W[n, k])) / Fraction(s)
            want = brute_force_code(float(v)) if v != 0 else (0x20 if np.signbit(W[n, k]) else 0)
            # float(v) is correctly rounded; w/s never sits within 2^-53 of a
            # midpoint unless it is one, so rounding the rational gives the same code
            assert codes[n, k] == want, (n, k, W[n, k], s)


def test_quantize_round_trip(orc):
    rng = np.random.default_rng(3)
    N, K = 16, 256
    codes = rng.integers(0, 64, size=(N, K), dtype=np.uint8)
    codes[:, 5] = np.where(rng.integers(0, 2, N) == 1, 0x1F, 0x3F)  # one +-28 per row
    scales_f = (2.0 ** rng.uniform(-12, 3, N)).astype(np.float16)
    t = orc.decode_table()
    W = (t[codes] * scales_f.astype(np.float64)[:, None]).astype(np.float32)
    assert np.array_equal(W.astype(np.float64), t[codes] * scales_f.astype(np.float64)[:, None])
    c2, s2 = orc.quantize(W)
    assert np.array_equal(s2, scales_f.view(np.uint16))
    # +0 and -0 both decode to zero; the sign of a zero weight is kept
    assert np.array_equal(c2, codes)


def test_quantize_special_rows(orc):
    W = np.zeros((3, 64), dtype=np.float32)
    W[1, :] = -0.0    # an all-zero row (negative zeros): scale 0, codes +0
    W[2, 0] = 28.0
    W[2, 1] = -1e-9   # rounds to zero, sign kept
    codes, scales = orc.quantize(W)
    assert scales[0] == 0 and not codes[0].any()
    assert scales[1] == 0 and not codes[1].any()
    assert scales[2] == np.float16(1.0).view(np.uint16)
    assert codes[2, 0] == 0x1F and codes[2, 1] == 0x20 and codes[2, 2] == 0


def test_quantize_errors(orc):
    W = np.ones((2, 64), dtype=np.float32)
    W[1, 3] = np.nan
    with pytest.raises(orc.OracleError) as e:
        orc.quantize(W)
    assert e.value.status == orc.ERR_NONFINITE
    W = np.ones((2, 64), dtype=np.float32)
    W[0, 0] = np.inf
    with pytest.raises(orc.OracleError):
        orc.quantize(W)
    W = np.ones((2, 64), dtype=np.float32)
    W[1, 0] = 3e6  # 3e6 / 28 > 65504
    with pytest.raises(orc.OracleError) as e:
        orc.quantize(W)
    assert e.value.status == orc.ERR_SCALE_RANGE
    W = np.zeros((1, 64), dtype=np.float32)
    W[0, 0] = 1e-10  # 1e-10 / 28 underflows fp16
    with pytest.raises(orc.OracleError) as e:
        orc.quantize(W)
    assert e.value.status == orc.ERR_SCALE_RANGE
