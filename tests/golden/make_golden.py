"""Writes tests/golden/e3m2_decode_table.txt from the oracle alone.

Run:  python tests/golden/make_golden.py
The file is a regression lock on the oracle's decode table; the independent
pin is the closed-form check in tests/test_oracle_decode.py.
"""
import os
import sys
from fractions import Fraction

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))
import oracle  # noqa: E402

with open(os.path.join(HERE, "e3m2_decode_table.txt"), "w") as f:
    f.write("# e3m2 FP6 decode table: code (hex) and exact value as a fraction.\n")
    f.write("# Format: sign/exponent(3, bias 3)/mantissa(2), no inf/NaN, max 28 (the layer's\n")
    f.write("# stated format; the FP6-LLM pages name only '6-bit float').\n")
    f.write("# Written by tests/golden/make_golden.py from oracle.decode_table().\n")
    for c, v in enumerate(oracle.decode_table()):
        f.write(f"0x{c:02x} {Fraction(v)}\n")
