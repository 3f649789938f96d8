"""Pins for the oracle's e3m2 decode table and its fp16 helpers.

The format (e3m2, exponent bias 3, no inf/NaN, max 28) is the layer's stated
specification; the FP6-LLM abstract and the TC-FPx article ("kernel solution
redesign") only say the weights are 6-bit floats turned into FP16 before the
tensor-core product.
"""
import os
from fractions import Fraction

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e3m2_decode_table.txt")


def closed_form(c: int) -> Fraction:
    s, e, m = (c >> 5) & 1, (c >> 2) & 7, c & 3
    if e == 0:
        mag = Fraction(1, 4) * Fraction(m, 4)
    else:
        mag = Fraction(2) ** (e - 3) * (1 + Fraction(m, 4))
    return -mag if s else mag


def test_decode_table_matches_closed_form_exhaustive(orc):
    t = orc.decode_table()
    for c in range(64):
        assert Fraction(t[c]) == closed_form(c), hex(c)


def test_decode_table_golden_file(orc):
    t = orc.decode_table()
    rows = [ln.split() for ln in open(GOLDEN) if ln.strip() and not ln.startswith("#")]
    assert len(rows) == 64
    for code_s, val_s in rows:
        c = int(code_s, 16)
        assert Fraction(t[c]) == Fraction(val_s), code_s


def test_decode_invariants(orc):
    t = orc.decode_table()
    # sign bit negates (including +0 / -0)
    for c in range(32):
        assert t[c | 0x20] == -t[c]
        assert np.signbit(t[c | 0x20]) != np.signbit(t[c]) or t[c] != 0
    # strictly increasing magnitudes over codes 0..31
    assert all(t[c] < t[c + 1] for c in range(31))
    assert t[0x1F] == 28.0 and t[0x04] == 0.25 and t[0x01] == 0.0625
    assert t[0x00] == 0.0 and np.signbit(t[0x20])


def test_splice_pattern_is_decode_times_2_pow_minus_12():
    """fp16 bits of decode(c) * 2^-12 equal (c & 0x20) << 10 | (c & 0x1F) << 8:
    the exponent field of the code sits unchanged in the low three bits of the
    fp16 exponent field, so the bit splice yields exact fp16 values (including
    the e3m2 subnormals, which land on fp16 subnormals)."""
    for c in range(64):
        v = float(closed_form(c)) * 2.0 ** -12
        if c & 0x20:
            v = -abs(v)  # code 0x20 is -0; Fraction has no signed zero
        bits = int(np.array([v], dtype=np.float64).astype(np.float16).view(np.uint16)[0])
        assert bits == (((c & 0x20) << 10) | ((c & 0x1F) << 8)), hex(c)


def test_f16_to_f64_all_patterns(orc):
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = pats.view(np.float16).astype(np.float64)
    got = np.array([orc.f16_to_f64(int(p)) for p in pats])
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(np.isinf(got), np.isinf(ref))


def test_f64_to_f16_rne_vs_numpy(orc):
    rng = np.random.default_rng(1)
    vals = []
    # random magnitudes over the whole fp16 range and beyond
    vals += list(rng.standard_normal(4000) * 10.0 ** rng.uniform(-9, 5, 4000))
    # every fp16 midpoint (ties) and its binary64 neighbours, sampled
    f16 = np.arange(0, 0x7BFF, 7, dtype=np.uint16).view(np.float16).astype(np.float64)
    nxt = np.arange(1, 0x7C00, 7, dtype=np.uint16).view(np.float16).astype(np.float64)
    mids = (f16 + nxt) / 2.0
    vals += list(mids) + list(np.nextafter(mids, 0)) + list(np.nextafter(mids, 1e9))
    vals += [65504.0, 65519.99, 65520.0, 70000.0, 2.0 ** -24, 2.0 ** -25, 2.0 ** -25 * 1.0000001,
             3 * 2.0 ** -26, 0.0, -0.0]
    vals = np.array(vals + [-v for v in vals], dtype=np.float64)
    ref = vals.astype(np.float16).view(np.uint16)
    got = orc.f64_to_f16_array(vals)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(vals[i], hex(got[i]), hex(ref[i])) for i in bad[:5]]
