"""Pins for the oracle's linear layer y = x . (s (.) decode(C))^T rounded to fp16.

The FP6-LLM abstract: weights are FP6, activations FP16 (W6A16); the TC-FPx
article: the FP6 weights are turned into FP16 and multiplied with the FP16
activations on tensor cores.  The plain definition therefore is an ordinary
matrix product of x with the reconstructed weights, rounded once to fp16.
"""
from fractions import Fraction

import numpy as np
import pytest

from tests.test_oracle_decode import closed_form

DEC = [closed_form(c) for c in range(64)]


def f16_frac(bits: int) -> Fraction:
    return Fraction(float(np.array([bits], dtype=np.uint16).view(np.float16)[0]))


def round_frac_to_f16(v: Fraction) -> int:
    """Exact round-to-nearest-even of a rational to fp16 (bit pattern)."""
    guess = np.array([float(v)], dtype=np.float64).astype(np.float16)
    cands = {int(guess.view(np.uint16)[0])}
    for d in (-1, 1):
        cands.add(int(np.nextafter(guess, np.float16(d * np.inf)).view(np.uint16)[0]))
    best = None
    for c in cands:
        fv = float(np.array([c], dtype=np.uint16).view(np.float16)[0])
        if not np.isfinite(fv):
            continue
        d = abs(Fraction(fv) - v)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c)
    return best[1]


def exact_linear(x16, codes, scales):
    M, K = x16.shape
    N = codes.shape[0]
    y = np.zeros((M, N), dtype=np.uint16)
    xf = [[f16_frac(int(b)) for b in row] for row in x16]
    for n in range(N):
        s = f16_frac(int(scales[n]))
        w = [s * DEC[int(c)] for c in codes[n]]
        for m in range(M):
            y[m, n] = round_frac_to_f16(sum((a * b for a, b in zip(xf[m], w)), Fraction(0)))
    return y


def rand_f16(rng, shape, lo_exp, hi_exp):
    """fp16 values with |x| in [2^lo_exp, 2^hi_exp) and random signs."""
    mag = 2.0 ** rng.uniform(lo_exp, hi_exp, size=shape)
    sgn = np.where(rng.integers(0, 2, size=shape) == 1, -1.0, 1.0)
    return (mag * sgn).astype(np.float16).view(np.uint16)


def test_linear_exact_rational_small_range(orc):
    """Operands chosen so that every partial sum is exact in binary64: the
    oracle must then equal the exactly rounded rational result bit for bit."""
    rng = np.random.default_rng(0)
    M, N, K = 3, 24, 64
    x = rand_f16(rng, (M, K), -6, 4)
    codes = rng.integers(0, 64, size=(N, K), dtype=np.uint8)
    scales = (2.0 ** rng.uniform(-8, 0, N)).astype(np.float16).view(np.uint16)
    assert np.array_equal(orc.linear(x, codes, scales), exact_linear(x, codes, scales))


def test_linear_exact_rational_general(orc):
    """N(0,1) activations and realistic codes: the double accumulation may
    round, so allow one fp16 ulp against the exact result (and require most to
    be equal)."""
    from weight_only_quantized_fp6_b200 import inputs
    W = inputs.weights(0, 16, 256)
    codes, scales = orc.quantize(W)
    x = inputs.activations(100, 2, 256)
    got = orc.linear(x, codes, scales)
    ref = exact_linear(x, codes, scales)
    diff = np.abs(got.view(np.int16).astype(np.int32) - ref.view(np.int16).astype(np.int32))
    assert diff.max() <= 1
    assert (diff == 0).mean() > 0.95


def test_linear_one_hot(orc):
    rng = np.random.default_rng(4)
    N, K = 64, 64
    codes = rng.integers(0, 64, size=(N, K), dtype=np.uint8)
    scales = (2.0 ** rng.uniform(-10, 4, N)).astype(np.float16)
    x = np.zeros((K, K), dtype=np.float16)
    x[np.arange(K), np.arange(K)] = 1.0
    y = orc.linear(x.view(np.uint16), codes, scales.view(np.uint16))
    vals = np.array([float(v) for v in DEC])
    want = (vals[codes].T * scales.astype(np.float64)[None, :]).astype(np.float16).view(np.uint16)
    nz = vals[codes].T != 0  # signed zero of the output is not part of the contract
    assert np.array_equal(y[nz], want[nz])
    assert not (y[~nz] & 0x7FFF).any()


def test_linear_constant_codes(orc):
    rng = np.random.default_rng(6)
    N, K, M = 64, 128, 4
    cvals = rng.integers(0, 64, size=N).astype(np.uint8)
    codes = np.repeat(cvals[:, None], K, axis=1)
    scales = np.full(N, np.float16(0.015625)).view(np.uint16)
    x = rand_f16(rng, (M, K), -4, 2)
    y = orc.linear(x, codes, scales)
    xs = [sum((f16_frac(int(b)) for b in row), Fraction(0)) for row in x]
    for n in range(N):
        for m in range(M):
            want = round_frac_to_f16(DEC[int(cvals[n])] * Fraction(1, 64) * xs[m])
            if (want & 0x7FFF) == 0:
                assert (int(y[m, n]) & 0x7FFF) == 0
            else:
                assert int(y[m, n]) == want


def test_linear_zero_input(orc):
    rng = np.random.default_rng(8)
    codes = rng.integers(0, 64, size=(32, 64), dtype=np.uint8)
    scales = np.full(32, np.float16(1.0)).view(np.uint16)
    y = orc.linear(np.zeros((2, 64), dtype=np.uint16), codes, scales)
    assert not (y & 0x7FFF).any()


def test_linear_threads_agree(orc):
    from weight_only_quantized_fp6_b200 import inputs
    W = inputs.weights(1, 128, 512)
    codes, scales = orc.quantize(W)
    x = inputs.activations(7, 5, 512)
    assert np.array_equal(orc.linear(x, codes, scales, 1), orc.linear(x, codes, scales, 4))


def test_linear_empty_shapes(orc):
    codes = np.zeros((8, 64), dtype=np.uint8)
    scales = np.zeros(8, dtype=np.uint16)
    assert orc.linear(np.zeros((0, 64), dtype=np.uint16), codes, scales).shape == (0, 8)
    y = orc.linear(np.zeros((3, 0), dtype=np.uint16), np.zeros((8, 0), dtype=np.uint8), scales)
    assert y.shape == (3, 8) and not (y & 0x7FFF).any()
