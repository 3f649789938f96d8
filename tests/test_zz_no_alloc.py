"""fp6_linear_noalloc: the layer for callers that cannot allocate device memory
while it runs (an engine plugin that does not own device memory, or a loop
where cudaMalloc's possible device synchronization is not allowed).  Its
scratch is a fixed array inside the library, so the test calls it through the
C ABI with no workspace and checks it against the CPU oracle (on every output,
or on sampled rows for the full-size layer) and against fp6_linear with a
workspace, on two calls in a row.

This file is collected last on purpose; it must pass on its own in a fresh
process as well as after the other tests.
"""
import ctypes

import numpy as np
import pytest

from tests import parity

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

SCRATCH_BYTES = 16 << 20


@pytest.fixture(scope="module")
def fp6():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from weight_only_quantized_fp6_b200 import build
    build.build_library()
    import weight_only_quantized_fp6_b200 as m
    return m


def bits16(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def call_noalloc(fp6, x, packed, scales, N, K, y):
    from weight_only_quantized_fp6_b200 import _lib
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return _lib.load().fp6_linear_noalloc(x.data_ptr(), packed.data_ptr(), scales.data_ptr(),
                                          x.shape[0], N, K, y.data_ptr(), stream)


@pytest.mark.parametrize("N,K,M", [(256, 512, 4), (1280, 4096, 1), (8192, 8192, 16), (640, 4096, 40),
                                   (8192, 8192, 64)])
def test_noalloc_matches_oracle_twice(fp6, orc, N, K, M):
    from weight_only_quantized_fp6_b200 import inputs
    W = inputs.weights(N + K + M, N, K)
    layer = fp6.FP6Linear.from_float(torch.from_numpy(W).cuda())
    x_np = inputs.activations(M * 7 + 1, M, K)
    x = torch.from_numpy(x_np.view(np.int16)).cuda().view(torch.float16)
    assert fp6.workspace_bytes(M, N, K) <= SCRATCH_BYTES
    # the oracle on every row of the small layers, on sampled rows of the 8192 x 8192 one
    rows = np.arange(N) if N * K <= 1280 * 4096 else parity.sample_rows(N, np.random.default_rng(N + M))
    codes_o, scales_o = orc.quantize(W[rows])
    ref = orc.linear(x_np, codes_o, scales_o, nthreads=16)
    with_ws = bits16(layer(x))
    for _ in range(2):  # two calls in a row share (and reuse) the fixed scratch
        y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        assert call_noalloc(fp6, x, layer.packed, layer.scales, N, K, y) == 0
        torch.cuda.synchronize()
        got = bits16(y)
        parity.assert_close(got[:, rows], ref, f"noalloc N={N} K={K} M={M}")
        assert np.array_equal(got, with_ws)  # same kernel, same summation order: identical bits
    assert fp6.device_status() == 0


@pytest.mark.parametrize("M", [65, 256])
def test_noalloc_rejects_problems_beyond_its_scratch(fp6, M):
    N, K = 8192, 8192  # M > 64 takes the wide token tiles, whose scratch exceeds 16 MiB here
    assert fp6.workspace_bytes(M, N, K) > SCRATCH_BYTES
    packed = torch.zeros(N * K * 3 // 4, dtype=torch.uint8, device="cuda")
    scales = torch.ones(N, dtype=torch.float16, device="cuda")
    x = torch.zeros((M, K), dtype=torch.float16, device="cuda")
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    assert call_noalloc(fp6, x, packed, scales, N, K, y) == 6  # FP6_ERR_WORKSPACE
