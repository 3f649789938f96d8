"""Seeded synthetic inputs shared by the tests, the oracle legs and the benchmark.

This module holds random-number generation only -- none of the layer's
arithmetic.  The generator is counter-based (splitmix64 finaliser over a
per-seed key plus the element index, then Box-Muller in binary64), so any row
range of a matrix can be regenerated on its own: the CPU oracle can rebuild a
few sampled rows of a large weight matrix without the rest.

Workloads (shapes of the Llama-70B and OPT-30B linear layers that the FP6-LLM
kernel evaluation used; no model weights are involved):
  * weights  W ~ N(0, 0.02) in fp32; OPT-shaped layers additionally multiply an
    independent Bernoulli(0.001) subset of weights by 8 (outliers);
  * activations x ~ N(0, 1) rounded to fp16 (round-to-nearest-even).
Seed scheme: weight seed = 1000 * config + layer index (the tiny case uses 0);
activation seed = weight seed + 100 + M.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_TWO_M53 = float(2.0 ** -53)
_CHUNK = 1 << 22


def _mix(z: np.ndarray) -> np.ndarray:
    """splitmix64 finaliser (wrapping uint64 arithmetic)."""
    z = z.copy()
    z ^= z >> np.uint64(30)
    z *= _M1
    z ^= z >> np.uint64(27)
    z *= _M2
    z ^= z >> np.uint64(31)
    return z


def _key(seed: int, stream: int) -> np.uint64:
    with np.errstate(over="ignore"):
        return _mix(np.array([np.uint64(seed) * np.uint64(4) + np.uint64(stream)], dtype=np.uint64))[0]


def _uniform(key: np.uint64, idx: np.ndarray, salt: int) -> np.ndarray:
    """53-bit uniform in [0, 1) for element indices idx."""
    with np.errstate(over="ignore"):
        z = key + (idx * np.uint64(3) + np.uint64(salt)) * _GOLDEN
        return (_mix(z) >> np.uint64(11)).astype(np.float64) * _TWO_M53


def normal_f64(seed: int, start: int, count: int, stream: int = 0) -> np.ndarray:
    """N(0,1) samples for flat element indices [start, start+count)."""
    key = _key(seed, stream)
    idx = np.arange(start, start + count, dtype=np.uint64)
    u1 = 1.0 - _uniform(key, idx, 0)          # (0, 1]
    u2 = _uniform(key, idx, 1)
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


def bernoulli(seed: int, start: int, count: int, p: float, stream: int = 2) -> np.ndarray:
    key = _key(seed, stream)
    idx = np.arange(start, start + count, dtype=np.uint64)
    return _uniform(key, idx, 2) < p


def weights(seed: int, N: int, K: int, rows=None, sigma: float = 0.02,
            outlier_p: float = 0.0, outlier_mult: float = 8.0, out=None) -> np.ndarray:
    """fp32 weight rows. rows = None (all N) or an iterable of row indices."""
    row_list = range(N) if rows is None else list(rows)
    n_out = len(row_list)
    W = out if out is not None else np.empty((n_out, K), dtype=np.float32)
    # Contiguous row runs are generated in chunks to bound memory.
    i = 0
    rl = list(row_list) if rows is not None else None
    while i < n_out:
        r0 = i if rl is None else rl[i]
        j = i + 1
        while j < n_out and (rl is None or rl[j] == rl[j - 1] + 1) and (j - i) * K < _CHUNK:
            j += 1
        cnt = (j - i) * K
        z = normal_f64(seed, r0 * K, cnt)
        w = (sigma * z).astype(np.float32)
        if outlier_p > 0.0:
            sel = bernoulli(seed, r0 * K, cnt, outlier_p)
            w[sel] *= np.float32(outlier_mult)
        W[i:j] = w.reshape(j - i, K)
        i = j
    return W


def weights_parallel(seed: int, N: int, K: int, outlier_p: float = 0.0, threads: int = 0) -> np.ndarray:
    """The full fp32 weight matrix, generated in row blocks on several threads
    (identical to weights(seed, N, K, outlier_p=...))."""
    W = np.empty((N, K), dtype=np.float32)
    threads = threads or min(16, os.cpu_count() or 4)
    block = max(1, N // (threads * 4))

    def job(r0):
        r1 = min(N, r0 + block)
        weights(seed, N, K, rows=range(r0, r1), outlier_p=outlier_p, out=W[r0:r1])

    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(job, range(0, N, block)))
    return W


def activations(seed: int, M: int, K: int) -> np.ndarray:
    """x ~ N(0,1) rounded to fp16; returned as fp16 bit patterns (uint16)."""
    z = normal_f64(seed, 0, M * K, stream=1)
    return z.astype(np.float16).view(np.uint16).reshape(M, K)


# ---- workload catalogue ------------------------------------------------------

LLAMA70B = {"qkv": (10240, 8192), "o": (8192, 8192), "gate_up": (57344, 8192), "down": (8192, 28672)}
OPT30B = {"qkv": (21504, 7168), "o": (7168, 7168), "fc1": (28672, 7168), "fc2": (7168, 28672)}
PREFILL = {"up": (28672, 8192), "down": (8192, 28672)}

# Workloads by name: layer shapes, token counts, outlier rate, and the base of
# the weight seeds of their layers (layer i of a workload draws its weights
# from seed_base + i).
WORKLOADS = {
    "tiny": {"layers": {"tiny": (256, 512)}, "M": [4], "outliers": 0.0, "seed_base": 0},
    "llama70b_o_decode": {"layers": {"o": LLAMA70B["o"]}, "M": [1, 2, 4, 8, 16], "outliers": 0.0,
                          "seed_base": 2000},
    "llama70b_all": {"layers": LLAMA70B, "M": [1, 4, 8, 16, 32], "outliers": 0.0, "seed_base": 3000},
    "opt30b": {"layers": OPT30B, "M": [1, 16, 64, 128], "outliers": 0.001, "seed_base": 4000},
    "prefill": {"layers": PREFILL, "M": [256, 1024, 4096], "outliers": 0.0, "seed_base": 5000},
}


def weight_seed(workload: str, layer_index: int) -> int:
    """Weight seed of layer `layer_index` of a named workload (the tiny
    workload's single layer uses seed 0)."""
    base = WORKLOADS[workload]["seed_base"]
    return base if base == 0 else base + layer_index


def activation_seed(wseed: int, M: int) -> int:
    return wseed + 100 + M
