"""Column-parallel split on the GPU, ranks emulated one after another on one
device: each rank's fp6_linear on its own slice of the packed weight gives its
output columns, and together they match the oracle for the whole layer."""
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


@pytest.mark.parametrize("world,N,K,M", [(2, 1280, 4096, 1), (3, 1280, 4096, 16), (4, 640, 8192, 40),
                                          (8, 8192, 1024, 4)])
def test_shards_assemble_the_layer(fp6, orc, world, N, K, M):
    from weight_only_quantized_fp6_b200 import column_parallel as cp
    from weight_only_quantized_fp6_b200 import inputs
    W = inputs.weights(51, N, K)
    x = inputs.activations(52, M, K)
    layer = fp6.FP6Linear.from_float(torch.from_numpy(W).cuda())
    xd = torch.from_numpy(x.view(np.int16)).cuda().view(torch.float16)
    cols = []
    for r in range(world):
        p, s, n0, n1 = cp.shard_packed(layer.packed, layer.scales, N, K, world, r)
        cols.append(fp6.linear(xd, p.contiguous(), s.contiguous(), n1 - n0, K))
    y = torch.cat(cols, dim=1)
    torch.cuda.synchronize()
    codes, scales = orc.quantize(W)
    parity.assert_close(y.cpu().view(torch.int16).numpy().view(np.uint16), orc.linear(x, codes, scales, nthreads=8),
                        f"world={world} N={N} K={K} M={M}")
