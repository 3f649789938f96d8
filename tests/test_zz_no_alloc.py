"""fp6_linear_noalloc: the layer for callers that cannot allocate device memory
while it runs (an engine plugin that does not own device memory, or a loop
where cudaMalloc's possible device synchronization is not allowed).  Its
scratch is a fixed array inside the library, so the test calls it through the
C ABI with no workspace and checks it against fp6_linear with a workspace.

This file is collected last on purpose; it must pass on its own in a fresh
process as well as after the other tests.
"""
import ctypes

import numpy as np
import pytest

from tests import parity

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


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


@pytest.mark.parametrize("N,K,M", [(256, 512, 4), (1280, 4096, 1), (8192, 8192, 16), (640, 4096, 40)])
def test_noalloc_matches_linear_twice(fp6, N, K, M):
    from weight_only_quantized_fp6_b200 import inputs
    W = torch.from_numpy(inputs.weights(N + K + M, N, K)).cuda()
    layer = fp6.FP6Linear.from_float(W)
    x = torch.from_numpy(inputs.activations(M * 7 + 1, M, K).view(np.int16)).cuda().view(torch.float16)
    ref = bits16(layer(x))
    for _ in range(2):  # two calls in a row share (and reuse) the fixed scratch
        y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        assert call_noalloc(fp6, x, layer.packed, layer.scales, N, K, y) == 0
        torch.cuda.synchronize()
        got = bits16(y)
        parity.assert_close(got, ref, f"noalloc N={N} K={K} M={M}")
        assert np.array_equal(got, ref)  # same kernel, same order: identical bits
    assert fp6.device_status() == 0


def test_noalloc_rejects_problems_beyond_its_scratch(fp6):
    N, K, M = 8192, 8192, 256  # needs a much larger split-K scratch than 16 MiB
    assert fp6.workspace_bytes(M, N, K) > (16 << 20)
    packed = torch.zeros(N * K * 3 // 4, dtype=torch.uint8, device="cuda")
    scales = torch.ones(N, dtype=torch.float16, device="cuda")
    x = torch.zeros((M, K), dtype=torch.float16, device="cuda")
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    assert call_noalloc(fp6, x, packed, scales, N, K, y) == 6  # FP6_ERR_WORKSPACE
