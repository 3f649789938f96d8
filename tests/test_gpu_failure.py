"""Failure detection on the GPU without a fault: a kernel waits on an mbarrier
that nothing arrives on.  The library's bounded wait must give up, report
FP6_ERR_TIMEOUT through the device error word, clear it when read, and leave
the context usable for the next fp6_linear call."""
import ctypes

import numpy as np
import pytest

from tests import parity

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

FP6_OK, FP6_ERR_TIMEOUT = 0, 9


@pytest.fixture(scope="module")
def fp6():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from weight_only_quantized_fp6_b200 import build
    build.build_library()
    import weight_only_quantized_fp6_b200 as m
    return m


def test_bounded_wait_times_out_and_context_survives(fp6, orc):
    from weight_only_quantized_fp6_b200 import _lib, inputs
    lib = _lib.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.fp6_get_device_status(stream) == FP6_OK
    assert lib.fp6_selftest_wait_timeout(stream) == FP6_OK
    torch.cuda.synchronize()                       # the kernel returns on its own
    assert lib.fp6_get_device_status(stream) == FP6_ERR_TIMEOUT
    assert lib.fp6_get_device_status(stream) == FP6_OK   # read-and-clear
    # the context is still usable: a normal layer call matches the oracle
    N, K, M = 256, 512, 4
    W = inputs.weights(7, N, K)
    x = inputs.activations(8, M, K)
    layer = fp6.FP6Linear.from_float(torch.from_numpy(W).cuda())
    y = layer(torch.from_numpy(x.view(np.int16)).cuda().view(torch.float16))
    torch.cuda.synchronize()
    codes, scales = orc.quantize(W)
    parity.assert_close(y.cpu().view(torch.int16).numpy().view(np.uint16), orc.linear(x, codes, scales),
                        "after a timed-out wait")
    assert lib.fp6_get_device_status(stream) == FP6_OK
