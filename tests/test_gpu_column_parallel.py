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


_NCCL_CHILD = r"""
import datetime, os, sys
import numpy as np, torch, torch.distributed as dist
sys.path.insert(0, os.environ["REPO"])
import oracle
import weight_only_quantized_fp6_b200 as fp6
from weight_only_quantized_fp6_b200 import inputs
from weight_only_quantized_fp6_b200.column_parallel import ColumnParallelFP6Linear
from tests import parity
torch.cuda.set_device(0)
dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                        device_id=torch.device("cuda", 0))
N, K, M = 1280, 2048, 24
fmt = None if os.environ["FMT"] == "none" else int(os.environ["FMT"])
W = inputs.weights(61, N, K)
x = inputs.activations(62, M, K)
full = fp6.FP6Linear.from_float(torch.from_numpy(W).cuda(), fmt=fmt)
layer = ColumnParallelFP6Linear(full.packed, full.scales, N, K, fmt=fmt)
xd = torch.from_numpy(x.view(np.int16)).cuda().view(torch.float16)
y = layer(xd)                                   # local product, then the NCCL all-gather
assert tuple(y.shape) == (M, N)
yl = layer(xd, gather=False)
assert torch.equal(y.view(torch.int16), yl.view(torch.int16))
bits = y.cpu().view(torch.int16).numpy().view(np.uint16)
if fmt == 4:
    q, pos, s = oracle.s24_quantize(W)
    ref = oracle.s24_linear(x, q, pos, s)
elif fmt is None:
    codes, s = oracle.quantize(W)
    ref = oracle.linear(x, codes, s, nthreads=8)
else:
    codes, s = oracle.fpx_quantize(fmt, W)
    ref = oracle.fpx_linear(fmt, x, codes, s)
parity.assert_close(bits, ref, "column-parallel, one NCCL rank")
assert fp6.device_status() == 0
dist.destroy_process_group()
print("ok")
"""


@pytest.mark.parametrize("fmt", ["none", "2", "4"])
def test_product_class_under_nccl(fp6, orc, fmt):
    """ColumnParallelFP6Linear as a caller uses it: a one-rank NCCL process
    group (this run has one GPU), the layer built from the full packed weight,
    __call__ with the all-gather, against the oracle.  Run in a child process
    so the process group lives and dies with it."""
    import os
    import socket
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    env = dict(os.environ, REPO=root, FMT=fmt, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
               NCCL_NVLS_ENABLE="0")
    out = subprocess.run([sys.executable, "-c", _NCCL_CHILD], env=env, cwd=root, capture_output=True,
                         text=True, timeout=300)
    assert out.returncode == 0 and out.stdout.strip().endswith("ok"), out.stdout[-2000:] + out.stderr[-2000:]
