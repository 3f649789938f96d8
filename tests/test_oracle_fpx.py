"""Pins for the oracle's other FPx formats: FP6 e2m3 (format 1), FP4 e2m1
(format 2) and FP5 e2m2 (format 3), each with one fp16 scale per output row.

The FP6-LLM abstract and the TC-FPx article present the kernel design as one
for float weights of several bit widths, without their bit formats.  The two
formats here follow the usual sign / exponent / mantissa reading:
  e2m3: s = bit 5, e = bits 4..3 (bias 1), m = bits 2..0, largest value 7.5;
  e2m1: s = bit 3, e = bits 2..1 (bias 1), m = bit 0,     largest value 6;
  e2m2: s = bit 4, e = bits 3..2 (bias 1), m = bits 1..0, largest value 7.
Every pin below is computed here from that definition, in exact rationals or
with numpy / CUDA library routines, never with the oracle's own code.
"""
import ctypes
import os
import shutil
import subprocess
from fractions import Fraction

import numpy as np
import pytest

FMTS = {1: dict(ebits=2, mbits=3, bias=1, maxv=Fraction(15, 2)),
        2: dict(ebits=2, mbits=1, bias=1, maxv=Fraction(6)),
        3: dict(ebits=2, mbits=2, bias=1, maxv=Fraction(7))}
ALL = [1, 2, 3]


def closed_form(fmt, c):
    f = FMTS[fmt]
    eb, mb, b = f["ebits"], f["mbits"], f["bias"]
    s = (c >> (eb + mb)) & 1
    e = (c >> mb) & ((1 << eb) - 1)
    m = c & ((1 << mb) - 1)
    frac = Fraction(m, 1 << mb)
    mag = (1 + frac) * Fraction(2) ** (e - b) if e > 0 else frac * Fraction(2) ** (1 - b)
    return -mag if s else mag


def closed_float(fmt, c):
    """closed_form as a binary64 value, keeping the sign of zero."""
    f = FMTS[fmt]
    neg = (c >> (f["ebits"] + f["mbits"])) & 1
    v = float(abs(closed_form(fmt, c)))
    return -v if neg else v


def ncodes(fmt):
    f = FMTS[fmt]
    return 1 << (1 + f["ebits"] + f["mbits"])


def mags(fmt):
    return [closed_form(fmt, c) for c in range(ncodes(fmt) // 2)]


@pytest.mark.parametrize("fmt", ALL)
def test_decode_table_closed_form(orc, fmt):
    t = orc.fpx_decode_table(fmt)
    assert len(t) == ncodes(fmt)
    for c in range(ncodes(fmt)):
        assert Fraction(t[c]) == closed_form(fmt, c), (fmt, c)
    assert Fraction(t[ncodes(fmt) // 2 - 1]) == FMTS[fmt]["maxv"]


def test_fp4_values_are_the_eight_e2m1_magnitudes(orc):
    assert [Fraction(v) for v in orc.fpx_decode_table(2)[:8]] == \
        [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3), Fraction(4), Fraction(6)]


def test_format_0_is_e3m2(orc):
    assert np.array_equal(orc.fpx_decode_table(0), orc.decode_table())
    for v in [0.0, 0.03, 0.09, 0.2, 1.1, 1.125, 2.5, 27.0, 29.9, 1e9, -3.3]:
        assert orc.fpx_round(0, v) == orc.round_e3m2(v)


def brute_force_code(fmt, v):
    """argmin over the format's magnitudes of |v| - mag, ties to the even code,
    saturating; sign copied from v."""
    a = abs(Fraction(v))
    best, bestd = None, None
    for c, mag in enumerate(mags(fmt)):
        d = abs(a - mag)
        if bestd is None or d < bestd or (d == bestd and c % 2 == 0):
            best, bestd = c, d
    sign = (ncodes(fmt) // 2) if np.signbit(v) else 0
    return sign | best


def probe_values(fmt):
    rng = np.random.default_rng(11 + fmt)
    m = [float(x) for x in mags(fmt)]
    mids = [(m[i] + m[i + 1]) / 2 for i in range(len(m) - 1)] + [float(FMTS[fmt]["maxv"]) * 1.1]
    vals = []
    for x in mids + m:
        vals += [x, float(np.nextafter(x, 0)), float(np.nextafter(x, 100))]
    top = float(FMTS[fmt]["maxv"])
    vals += list(rng.uniform(0, 1.5 * top, 3000)) + list(rng.uniform(0, 0.6, 1000))
    vals += [0.0, 1e-300, top, top * 1.2, 1e30]
    return vals + [-v for v in vals]


@pytest.mark.parametrize("fmt", ALL)
def test_round_vs_brute_force(orc, fmt):
    for v in probe_values(fmt):
        assert orc.fpx_round(fmt, v) == brute_force_code(fmt, v), (fmt, v)


@pytest.fixture(scope="module")
def cuda_cvt(tmp_path_factory):
    """CUDA's own host-side double -> e2m3 / e2m1 conversions (cuda_fp6.h,
    cuda_fp4.h), called as library routines for a second opinion."""
    inc = "/usr/local/cuda/include"
    if not os.path.exists(os.path.join(inc, "cuda_fp4.h")) or shutil.which("g++") is None:
        pytest.skip("cuda_fp4.h / cuda_fp6.h or g++ unavailable")
    d = tmp_path_factory.mktemp("fpxcvt")
    src = d / "cvt.cpp"
    src.write_text('#include <cuda_fp6.h>\n#include <cuda_fp4.h>\n'
                   'extern "C" unsigned char cvt6(double x){'
                   'return (unsigned char)__nv_cvt_double_to_fp6(x, __NV_E2M3, cudaRoundNearest);}\n'
                   'extern "C" unsigned char cvt4(double x){'
                   'return (unsigned char)__nv_cvt_double_to_fp4(x, __NV_E2M1, cudaRoundNearest);}\n')
    so = d / "cvt.so"
    subprocess.run(["g++", "-O1", "-shared", "-fPIC", "-I" + inc, str(src), "-o", str(so)], check=True)
    lib = ctypes.CDLL(str(so))
    for fn in (lib.cvt6, lib.cvt4):
        fn.argtypes = [ctypes.c_double]
        fn.restype = ctypes.c_uint8
    return {1: lib.cvt6, 2: lib.cvt4}


@pytest.mark.parametrize("fmt", [1, 2])
def test_round_vs_cuda_library(orc, cuda_cvt, fmt):
    for v in probe_values(fmt):
        assert orc.fpx_round(fmt, v) == cuda_cvt[fmt](v), (fmt, v)


@pytest.mark.parametrize("fmt", ALL)
def test_quantize_scale_and_codes(orc, fmt):
    from weight_only_quantized_fp6_b200 import inputs
    W = inputs.weights(21 + fmt, 128, 128)
    codes, scales = orc.fpx_quantize(fmt, W)
    amax = np.abs(W).max(axis=1).astype(np.float32)
    ref = (amax / np.float32(float(FMTS[fmt]["maxv"]))).astype(np.float16).view(np.uint16)
    assert np.array_equal(scales, ref)
    s = scales.view(np.float16).astype(np.float64)
    for n in range(0, 128, 9):
        for k in range(0, 128, 7):
            q = Fraction(float(W[n, k])) / Fraction(float(s[n]))
            assert codes[n, k] == brute_force_code(fmt, float(q)) or \
                codes[n, k] == brute_force_code(fmt, float(np.float64(W[n, k]) / s[n])), (n, k)


@pytest.mark.parametrize("fmt", ALL)
def test_quantize_round_trip(orc, fmt):
    """Rows built from codes (one at the largest magnitude each) times a
    power-of-two scale come back with the same codes and scale."""
    rng = np.random.default_rng(5)
    N, K = 16, 64
    nc = ncodes(fmt)
    codes = rng.integers(0, nc, size=(N, K)).astype(np.uint8)
    codes[:, 3] = nc // 2 - 1                     # +max in every row
    table = np.array([closed_float(fmt, c) for c in range(nc)])
    s = 2.0 ** rng.integers(-6, 3, size=N)
    W = (table[codes] * s[:, None]).astype(np.float32)
    c2, s2 = orc.fpx_quantize(fmt, W)
    zero = (table[codes] == 0)
    # codes of zero weights come back as +0 or -0 according to their sign
    assert np.array_equal(c2[~zero], codes[~zero])
    assert np.array_equal(s2.view(np.float16).astype(np.float64), s)


def read_fp4_codes(packed, N, K):
    """Independent reader of the FP4 layout: 4096-byte tiles, row r of a tile
    in words (w/4)*2048 + r*16 + (w%4)*4, column kk in word kk/8, byte
    (kk%8)/2, low nibble for even kk."""
    words = packed.view("<u4")
    out = np.zeros((N, K), dtype=np.uint8)
    KT = K // 64
    r = np.arange(128)
    for nt in range(N // 128):
        for kt in range(KT):
            base = (nt * KT + kt) * 1024
            for kk in range(64):
                w = kk // 8
                word = words[base + (w // 4) * 512 + r * 4 + (w % 4)]
                shift = 8 * ((kk % 8) // 2) + 4 * (kk % 2)
                out[nt * 128:(nt + 1) * 128, kt * 64 + kk] = (word >> shift) & 0xF
    return out


def test_fp4_prepack_reader_and_round_trip(orc):
    rng = np.random.default_rng(3)
    N, K = 256, 192
    codes = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    packed = orc.fpx_prepack(2, codes)
    assert packed.size == N * K // 2 == orc.fpx_packed_bytes(2, N, K)
    assert np.array_equal(read_fp4_codes(packed, N, K), codes)
    assert np.array_equal(orc.fpx_unpack(2, packed, N, K), codes)


def test_fp4_one_hot_probe(orc):
    N, K = 128, 128
    for (n, k) in [(0, 0), (0, 1), (5, 63), (127, 64), (64, 127), (77, 9)]:
        codes = np.zeros((N, K), dtype=np.uint8)
        codes[n, k] = 0xF
        packed = orc.fpx_prepack(2, codes)
        nz = np.nonzero(packed)[0]
        assert len(nz) == 1
        b = nz[0]
        tile = b // 4096
        assert tile == (n // 128) * (K // 64) + k // 64
        kk = k % 64
        assert (b % 4096) == ((kk // 8) // 4) * 2048 + (n % 128) * 16 + ((kk // 8) % 4) * 4 + (kk % 8) // 2
        assert packed[b] == (0x0F if kk % 2 == 0 else 0xF0)


def test_e2m3_uses_the_six_bit_layout(orc):
    rng = np.random.default_rng(4)
    codes = rng.integers(0, 64, size=(128, 128)).astype(np.uint8)
    assert np.array_equal(orc.fpx_prepack(1, codes), orc.prepack(codes))


@pytest.mark.parametrize("fmt", ALL)
def test_dequant_closed_form(orc, fmt):
    rng = np.random.default_rng(8)
    N, K = 128, 128
    codes = rng.integers(0, ncodes(fmt), size=(N, K)).astype(np.uint8)
    scales = (rng.uniform(0.01, 2.0, N)).astype(np.float16).view(np.uint16)
    packed = orc.fpx_prepack(fmt, codes)
    table = np.array([closed_float(fmt, c) for c in range(ncodes(fmt))])
    ref = (table[codes] * scales.view(np.float16).astype(np.float64)[:, None]).astype(np.float16).view(np.uint16)
    assert np.array_equal(orc.fpx_dequant(fmt, packed, scales, N, K), ref)
    ref1 = table[codes].astype(np.float16).view(np.uint16)
    assert np.array_equal(orc.fpx_dequant(fmt, packed, None, N, K), ref1)


@pytest.mark.parametrize("fmt", ALL)
def test_linear_exact_rational(orc, fmt):
    """Tiny shapes: the sum done in exact rationals, rounded once to fp16."""
    rng = np.random.default_rng(9 + fmt)
    M, N, K = 3, 8, 48
    codes = rng.integers(0, ncodes(fmt), size=(N, K)).astype(np.uint8)
    scales = rng.uniform(0.01, 1.0, N).astype(np.float16).view(np.uint16)
    x = rng.standard_normal((M, K)).astype(np.float16).view(np.uint16)
    y = orc.fpx_linear(fmt, x, codes, scales)
    xf = x.view(np.float16)
    sf = scales.view(np.float16)
    for m in range(M):
        for n in range(N):
            acc = sum(Fraction(float(xf[m, k])) * Fraction(float(sf[n])) * closed_form(fmt, int(codes[n, k]))
                      for k in range(K))
            want = np.float16(float(acc))
            got = y[m, n:n + 1].view(np.float16)[0]
            # binary64 summation may differ from the exact sum by far less than
            # an fp16 ulp; allow the one-ulp case of a near-tie
            assert got == want or abs(float(got) - float(want)) <= abs(float(want)) * 2.0 ** -10, (m, n)


@pytest.mark.parametrize("fmt", ALL)
def test_linear_one_hot(orc, fmt):
    rng = np.random.default_rng(12)
    N, K = 16, 64
    codes = rng.integers(0, ncodes(fmt), size=(N, K)).astype(np.uint8)
    scales = rng.uniform(0.01, 1.0, N).astype(np.float16).view(np.uint16)
    x = np.zeros((K, K), dtype=np.float16)
    np.fill_diagonal(x, 1.0)
    y = orc.fpx_linear(fmt, x.view(np.uint16), codes, scales)
    table = np.array([closed_float(fmt, c) for c in range(ncodes(fmt))])
    ref = (table[codes].T * scales.view(np.float16).astype(np.float64)[None, :]).astype(np.float16)
    # values compared (an empty sum of signed zeros is +0: the sign of a zero output is not pinned)
    assert np.array_equal(y.view(np.float16), ref)


def test_fp5_values_are_e2m3_values_via_cuda(orc, cuda_cvt):
    """Every e2m2 value is the e2m3 value of the code shifted left by one (the
    mantissa gains a zero bit): CUDA's own e2m3 conversion of each e2m2 value
    returns exactly that code."""
    t = orc.fpx_decode_table(3)
    for c in range(32):
        assert Fraction(t[c]) == closed_form(3, c)
        if closed_form(3, c) != 0:
            assert cuda_cvt[1](float(t[c])) == ((c & 0x10) << 1) | ((c & 0x0F) << 1), c


def read_fp5_codes(packed, N, K):
    """Independent reader of the FP5 layout, word by word as a GPU thread reads
    a row: eight 4-bit-piece words P_w at (w/4)*2048 + r*16 + (w%4)*4 and two
    1-bit-piece words Q_q at 4096 + r*8 + q*4 in each 5120-byte tile.  For
    word P_{4q+v}: byte b holds the pieces of codes b (low nibble) and b+4
    (high nibble) of its group of eight; their low bits are Q_q bits
    8b+2v and 8b+2v+1."""
    words = packed.view("<u4")
    out = np.zeros((N, K), dtype=np.uint8)
    KT = K // 64
    r = np.arange(128)
    for nt in range(N // 128):
        for kt in range(KT):
            base = (nt * KT + kt) * 1280                     # words per tile
            for q in range(2):
                Q = words[base + 1024 + r * 2 + q]
                for v in range(4):
                    w = 4 * q + v
                    P = words[base + (w // 4) * 512 + r * 4 + (w % 4)]
                    for h in range(2):
                        for b in range(4):
                            kk = 32 * q + 8 * v + 4 * h + b
                            top = (P >> (8 * b + 4 * h)) & 0xF
                            low = (Q >> (8 * b + 2 * v + h)) & 1
                            out[nt * 128:(nt + 1) * 128, kt * 64 + kk] = (top << 1) | low
    return out


def test_fp5_prepack_reader_and_round_trip(orc):
    rng = np.random.default_rng(13)
    N, K = 256, 192
    codes = rng.integers(0, 32, size=(N, K)).astype(np.uint8)
    packed = orc.fpx_prepack(3, codes)
    assert packed.size == N * K * 5 // 8 == orc.fpx_packed_bytes(3, N, K)
    assert np.array_equal(read_fp5_codes(packed, N, K), codes)
    assert np.array_equal(orc.fpx_unpack(3, packed, N, K), codes)


def test_fp5_one_hot_probe(orc):
    """A code with only its low bit set touches one bit of a Q word; a code
    with only its top four bits set touches one nibble of a P word."""
    N, K = 128, 128
    for (n, k) in [(0, 0), (0, 1), (5, 63), (127, 64), (64, 127), (77, 9), (3, 36)]:
        t = (n // 128) * (K // 64) + k // 64
        kk = k % 64
        q, i = kk // 32, kk % 32
        v, h, b = i // 8, (i % 8) // 4, i % 4
        r = n % 128
        for code, want_off, want_val in [
                (0x01, 4096 + r * 8 + q * 4 + (8 * b + 2 * v + h) // 8, 1 << ((2 * v + h) % 8)),
                (0x1E, ((4 * q + v) // 4) * 2048 + r * 16 + ((4 * q + v) % 4) * 4 + b, 0xF << (4 * h))]:
            codes = np.zeros((N, K), dtype=np.uint8)
            codes[n, k] = code
            packed = orc.fpx_prepack(3, codes)
            nz = np.nonzero(packed)[0]
            assert list(nz) == [t * 5120 + want_off], (n, k, code)
            assert packed[nz[0]] == want_val, (n, k, code)
