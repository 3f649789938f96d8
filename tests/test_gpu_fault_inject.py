"""Host-side fault injection (FP6_FAULT_INJECT=<point>[:<count>]): the
library's error paths for a failed tensor-map encode, a failed launch and a
failed stream synchronisation report FP6_ERR_CUDA and leave the outputs
untouched; once the injected failures are used up the same process computes
the layer correctly.  Nothing faults, traps or hangs on the GPU: the failure
is made on the host.  Each case runs in a child process (the variable is read
once per process)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

_CHILD = r"""
import os, sys
import numpy as np, torch
sys.path.insert(0, os.environ["REPO"])
import weight_only_quantized_fp6_b200 as fp6
point = os.environ["FP6_FAULT_INJECT"].split(":")[0]
N, K, M = 256, 512, 4
W = torch.randn(N, K, device="cuda") * 0.02
if point == "sync":
    with __import__("pytest").raises(fp6.FP6Error) as e:
        fp6.quantize(W)
    assert e.value.status == 8
    layer = fp6.FP6Linear.from_float(W)          # the injection is used up: this one succeeds
else:
    layer = fp6.FP6Linear.from_float(W)
    x = torch.randn(M, K, device="cuda").half()
    y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
    for _ in range(2):                            # FP6_FAULT_INJECT=<point>:2
        try:
            layer(x, out=y)
            raise SystemExit("no error reported")
        except fp6.FP6Error as e:
            assert e.status == 8, e.status
    torch.cuda.synchronize()
    assert torch.isnan(y).all()                  # nothing was launched
    got = fp6.linear(x, layer.packed, layer.scales, N, K)   # injection used up
    import oracle
    from tests import parity
    codes, scales = oracle.quantize(W.cpu().numpy())
    xb = x.cpu().view(torch.int16).numpy().view(np.uint16)
    parity.assert_close(got.cpu().view(torch.int16).numpy().view(np.uint16), oracle.linear(xb, codes, scales),
                        "after injected failures")
assert fp6.device_status() == 0
print("ok")
"""


@pytest.mark.parametrize("spec", ["encode:2", "launch:2", "sync:1"])
def test_injected_host_failures(spec):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, REPO=root, FP6_FAULT_INJECT=spec)
    out = subprocess.run([sys.executable, "-c", _CHILD], env=env, cwd=root, capture_output=True, text=True,
                         timeout=300)
    assert out.returncode == 0 and out.stdout.strip().endswith("ok"), out.stdout[-2000:] + out.stderr[-2000:]
