"""Pins for the oracle's 2:4 sparse INT4 weights (the Sparse-Marlin format:
4-bit weights, two kept in every group of four, their positions as metadata,
one fp16 scale per output row).

Readings (the post fixes none of the details): magnitude pruning, the two
largest |w| of each group kept with ties going to the lower position; scale
s = fp16(fp32(max|w| / 7)); codes round(w / s) to nearest, ties to even,
clamped to [-8, 7].  Every pin below is computed here from those
definitions -- properties that fix the kept set uniquely, exact rationals,
numpy's float16 -- never with the oracle's own code.
"""
from fractions import Fraction

import numpy as np
import pytest


def groups(W):
    N, K = W.shape
    return W.reshape(N, K // 4, 4)


def kept_mask(pos, N, K):
    m = np.zeros((N, K // 4, 4), dtype=bool)
    p = pos.reshape(N, K // 4, 2)
    for a in range(2):
        np.put_along_axis(m, p[:, :, a:a + 1].astype(np.int64), True, axis=2)
    return m


def test_pruning_properties(orc):
    """Exactly two kept per group, in increasing position order; every kept
    |w| is >= every pruned |w| of its group; where a kept and a pruned entry
    have equal |w|, the kept one sits at the lower position.  Together these
    fix the kept pair uniquely."""
    rng = np.random.default_rng(1)
    N, K = 64, 256
    W = rng.standard_normal((N, K)).astype(np.float32)
    # ties: repeated magnitudes, signs, zeros
    W[:8] = rng.integers(-2, 3, size=(8, K)).astype(np.float32)
    W[8:12] = 0.0
    W[8:12, ::7] = 1.0
    W[12, :] = np.tile(np.array([1, -1, 1, -1], dtype=np.float32), K // 4)
    q, pos, s = orc.s24_quantize(W)
    p = pos.reshape(N, K // 4, 2)
    assert (p[:, :, 0] < p[:, :, 1]).all()
    assert (p <= 3).all()
    m = kept_mask(pos, N, K)
    assert (m.sum(axis=2) == 2).all()
    a = np.abs(groups(W))
    kept_min = np.where(m, a, np.inf).min(axis=2)
    pruned_max = np.where(~m, a, -np.inf).max(axis=2)
    assert (kept_min >= pruned_max).all()
    # tie rule
    for n in range(N):
        for j in range(K // 4):
            for i in range(4):
                if m[n, j, i]:
                    continue
                for i2 in range(4):
                    if m[n, j, i2] and a[n, j, i2] == a[n, j, i]:
                        assert i2 < i, (n, j, i, i2)


def brute_code(v: Fraction) -> int:
    """argmin over q in [-8, 7] of |v - q|, ties to the even q."""
    best = None
    for c in range(-8, 8):
        d = abs(v - c)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c)
    return best[1]


def test_scale_and_codes(orc):
    from weight_only_quantized_fp6_b200 import inputs
    W = inputs.weights(31, 128, 128)
    q, pos, s = orc.s24_quantize(W)
    amax = np.abs(W).max(axis=1).astype(np.float32)
    assert np.array_equal(s, (amax / np.float32(7.0)).astype(np.float16).view(np.uint16))
    sf = s.view(np.float16).astype(np.float64)
    for n in range(0, 128, 5):
        for g in range(0, 32, 3):
            for a in range(2):
                k = 4 * g + int(pos[n, 2 * g + a])
                want = brute_code(Fraction(float(W[n, k])) / Fraction(float(sf[n])))
                assert int(q[n, 2 * g + a]) == want, (n, g, a)


def test_round_trip_of_representable_rows(orc):
    """Rows holding s*q at two positions per group (others zero, one entry at
    7s) come back with the same codes, positions and scale."""
    rng = np.random.default_rng(2)
    N, K = 32, 64
    W = np.zeros((N, K), dtype=np.float32)
    want_q = np.zeros((N, K // 2), dtype=np.int8)
    want_pos = np.zeros((N, K // 2), dtype=np.uint8)
    s = 2.0 ** rng.integers(-8, 2, size=N)
    pairs = [(0, 1), (0, 2), (0, 3), (1, 2), (1, 3), (2, 3)]
    for n in range(N):
        for g in range(K // 4):
            i0, i1 = pairs[rng.integers(0, 6)]
            c = rng.choice([c for c in range(-7, 8) if c != 0], size=2)
            if n % 2 == 0 and g == 0:
                c[0] = 7
            want_q[n, 2 * g:2 * g + 2] = c
            want_pos[n, 2 * g:2 * g + 2] = (i0, i1)
            W[n, 4 * g + i0] = c[0] * s[n]
            W[n, 4 * g + i1] = c[1] * s[n]
        W[n, 4 * 5 + want_pos[n, 10]] = 7 * s[n]          # the row maximum is exactly 7 s
        want_q[n, 10] = 7
    q, pos, sc = orc.s24_quantize(W)
    assert np.array_equal(sc.view(np.float16).astype(np.float64), s)
    assert np.array_equal(pos, want_pos)
    assert np.array_equal(q, want_q)


def test_zero_row_and_errors(orc):
    W = np.zeros((2, 8), dtype=np.float32)
    W[1, 3] = 1.0
    q, pos, s = orc.s24_quantize(W)
    assert s[0] == 0 and (q[0] == 0).all()
    assert list(pos[0, :2]) == [0, 1]                       # all-zero group: ties keep the lowest two
    bad = W.copy()
    bad[0, 0] = np.nan
    with pytest.raises(Exception):
        orc.s24_quantize(bad)
    with pytest.raises(Exception):
        orc.s24_quantize(np.ones((2, 6), dtype=np.float32))  # K not a multiple of 4


def read_s24(packed, N, K):
    """Independent word-level reader of the packed layout: 3072-byte tiles,
    row r: code words at r*16 + 4w (w = 0..3), position words at
    2048 + r*8 + 4h (h = 0, 1); group j's codes in byte j%4 of word j/4,
    positions in nibble j%8 of position word j/8."""
    words = packed.view("<u4")
    q = np.zeros((N, K // 2), dtype=np.int8)
    pos = np.zeros((N, K // 2), dtype=np.uint8)
    KT = K // 64
    r = np.arange(128)
    for nt in range(N // 128):
        for kt in range(KT):
            base = (nt * KT + kt) * 768                     # words per tile
            for j in range(16):
                V = words[base + r * 4 + j // 4]
                P = words[base + 512 + r * 2 + j // 8]
                byte = (V >> (8 * (j % 4))) & 0xFF
                nib = (P >> (4 * (j % 8))) & 0xF
                lo, hi = byte & 0xF, byte >> 4
                g = kt * 16 + j
                rows = slice(nt * 128, (nt + 1) * 128)
                q[rows, 2 * g] = np.where(lo >= 8, lo.astype(np.int64) - 16, lo)
                q[rows, 2 * g + 1] = np.where(hi >= 8, hi.astype(np.int64) - 16, hi)
                pos[rows, 2 * g] = nib & 3
                pos[rows, 2 * g + 1] = nib >> 2
    return q, pos


def test_layout_reader_and_round_trip(orc):
    rng = np.random.default_rng(3)
    N, K = 256, 192
    q = rng.integers(-8, 8, size=(N, K // 2)).astype(np.int8)
    pairs = np.array([(0, 1), (0, 2), (0, 3), (1, 2), (1, 3), (2, 3)], dtype=np.uint8)
    pos = pairs[rng.integers(0, 6, size=(N, K // 4))].reshape(N, K // 2)
    packed = orc.s24_prepack(q, pos)
    assert packed.size == N * K * 3 // 8 == orc.s24_packed_bytes(N, K)
    rq, rp = read_s24(packed, N, K)
    assert np.array_equal(rq, q) and np.array_equal(rp, pos)
    uq, up = orc.s24_unpack(packed, N, K)
    assert np.array_equal(uq, q) and np.array_equal(up, pos)


def test_one_hot_probe(orc):
    """One nonzero code (and one nonzero position) touches exactly one nibble
    of the right word."""
    N, K = 128, 128
    for (n, g, a) in [(0, 0, 0), (0, 0, 1), (5, 15, 1), (127, 16, 0), (64, 31, 1), (77, 9, 0)]:
        q = np.zeros((N, K // 2), dtype=np.int8)
        pos = np.zeros((N, K // 2), dtype=np.uint8)
        q[n, 2 * g + a] = -1                                  # 0xF
        packed = orc.s24_prepack(q, pos)
        nz = np.nonzero(packed)[0]
        t = (n // 128) * (K // 64) + g // 16
        j = g % 16
        assert list(nz) == [t * 3072 + (n % 128) * 16 + 4 * (j // 4) + (j % 4)]
        assert packed[nz[0]] == (0x0F if a == 0 else 0xF0)
        q[n, 2 * g + a] = 0
        pos[n, 2 * g + a] = 3
        packed = orc.s24_prepack(q, pos)
        nz = np.nonzero(packed)[0]
        bit = 4 * (j % 8) + 2 * a
        assert list(nz) == [t * 3072 + 2048 + (n % 128) * 8 + 4 * (j // 8) + bit // 8]
        assert packed[nz[0]] == 3 << (bit % 8)


def test_dequant_closed_form(orc):
    rng = np.random.default_rng(4)
    N, K = 128, 128
    q = rng.integers(-8, 8, size=(N, K // 2)).astype(np.int8)
    pairs = np.array([(0, 1), (0, 2), (0, 3), (1, 2), (1, 3), (2, 3)], dtype=np.uint8)
    pos = pairs[rng.integers(0, 6, size=(N, K // 4))].reshape(N, K // 2)
    scales = rng.uniform(0.001, 2.0, N).astype(np.float16)
    packed = orc.s24_prepack(q, pos)
    dense = np.zeros((N, K), dtype=np.float64)
    for n in range(N):
        for g in range(K // 4):
            for a in range(2):
                dense[n, 4 * g + pos[n, 2 * g + a]] = q[n, 2 * g + a]
    ref = (dense * scales.astype(np.float64)[:, None]).astype(np.float16).view(np.uint16)
    got = orc.s24_dequant(packed, scales.view(np.uint16), N, K)
    # compare as values: zeros of negative products come out as +0 from the oracle
    assert np.array_equal(got.view(np.float16).astype(np.float64), ref.view(np.float16).astype(np.float64))
    assert np.array_equal(orc.s24_dequant(packed, None, N, K).view(np.float16).astype(np.float64), dense)


def test_linear_exact_rational(orc):
    rng = np.random.default_rng(5)
    M, N, K = 3, 8, 48
    W = rng.standard_normal((N, K)).astype(np.float32)
    q, pos, s = orc.s24_quantize(W)
    x = rng.standard_normal((M, K)).astype(np.float16).view(np.uint16)
    y = orc.s24_linear(x, q, pos, s)
    xf, sf = x.view(np.float16), s.view(np.float16)
    for m in range(M):
        for n in range(N):
            acc = Fraction(0)
            for g in range(K // 4):
                for a in range(2):
                    k = 4 * g + int(pos[n, 2 * g + a])
                    acc += Fraction(float(xf[m, k])) * Fraction(float(sf[n])) * int(q[n, 2 * g + a])
            want = np.float16(float(acc))
            got = y[m, n:n + 1].view(np.float16)[0]
            assert got == want or abs(float(got) - float(want)) <= abs(float(want)) * 2.0 ** -10, (m, n)


def test_linear_one_hot(orc):
    """x = unit rows: y[m, n] is the dequantized weight at column m."""
    rng = np.random.default_rng(6)
    N, K = 128, 64
    W = rng.standard_normal((N, K)).astype(np.float32)
    q, pos, s = orc.s24_quantize(W)
    x = np.zeros((K, K), dtype=np.float16)
    x[np.arange(K), np.arange(K)] = 1.0
    y = orc.s24_linear(x.view(np.uint16), q, pos, s)
    W16 = orc.s24_dequant(orc.s24_prepack(q, pos), s, N, K)
    assert np.array_equal(y.view(np.float16).astype(np.float64), W16.T.view(np.float16).astype(np.float64))


def test_rounding_ties_go_to_even(orc):
    """Values exactly halfway between two codes (s a power of two, so w / s
    is exact) round to the even code."""
    s = 2.0 ** -3
    halves = [k + 0.5 for k in range(-7, 7)]                 # -6.5 .. 6.5: the row maximum stays 7 s
    K = 4 * len(halves)
    W = np.zeros((1, K), dtype=np.float32)
    for g, h in enumerate(halves):
        W[0, 4 * g] = 7 * s if g == 0 else h * s            # group 0 fixes the scale at s
        W[0, 4 * g + 2] = h * s
    q, pos, sc = orc.s24_quantize(W)
    assert sc.view(np.float16)[0] == np.float16(s)
    for g, h in enumerate(halves):
        a = 1                                                # the entry at position 2
        assert int(pos[0, 2 * g + a]) == 2
        want = int(np.round(h))                              # numpy rounds halves to even
        assert int(q[0, 2 * g + a]) == want, (h, int(q[0, 2 * g + a]))
