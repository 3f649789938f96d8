"""Shared helpers for the GPU parity tests: seeded workloads, the comparison
rule, and oracle runs on sampled rows.

Comparison rule for the linear layer (the layer's stated tolerance):
    |y - ref| <= 2^-9 |ref| + 1e-3 rms(ref)   per element, no NaN/inf,
with rms over the compared elements of one (shape, M) case.  Quantize,
prepack and dequant are compared byte for byte.
"""
from __future__ import annotations

import numpy as np

from weight_only_quantized_fp6_b200 import inputs

REL = 2.0 ** -9
ABS_RMS = 1e-3


def f16(bits: np.ndarray) -> np.ndarray:
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def assert_close(y_bits: np.ndarray, ref_bits: np.ndarray, what: str = ""):
    y = f16(y_bits)
    ref = f16(ref_bits)
    assert np.isfinite(ref).all(), f"{what}: reference not finite"
    assert np.isfinite(y).all(), f"{what}: NaN/inf in output"
    rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0
    err = np.abs(y - ref)
    bound = REL * np.abs(ref) + ABS_RMS * rms
    bad = np.nonzero(err > bound)
    assert bad[0].size == 0, (
        f"{what}: {bad[0].size} elements out of tolerance; first at {tuple(b[0] for b in bad)}: "
        f"got {y[tuple(b[0] for b in bad)]} want {ref[tuple(b[0] for b in bad)]}")


def gen_weights_parallel(seed: int, N: int, K: int, outlier_p: float) -> np.ndarray:
    return inputs.weights_parallel(seed, N, K, outlier_p)


def sample_rows(N: int, rng: np.random.Generator, extra: int = 64) -> np.ndarray:
    """Two whole 128-row tiles (first and last) plus random rows."""
    rows = set(range(0, 128)) | set(range(N - 128, N))
    rows |= set(int(r) for r in rng.integers(0, N, extra))
    return np.array(sorted(rows), dtype=np.int64)


def sample_tokens(M: int, rng: np.random.Generator, limit: int = 32) -> np.ndarray:
    if M <= limit:
        return np.arange(M)
    rest = rng.choice(np.arange(1, M - 1), size=limit - 2, replace=False)
    return np.array(sorted({0, M - 1} | set(int(v) for v in rest)), dtype=np.int64)
