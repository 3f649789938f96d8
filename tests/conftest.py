import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(autouse=True)
def no_device_error_left(request):
    """After every GPU test: the library's device error word (bounded waits
    that gave up) must be clear, so a silent timeout is pinned to the test
    that caused it."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    import torch
    if not torch.cuda.is_available():
        return
    from weight_only_quantized_fp6_b200 import _lib
    if _lib._lib is None:       # the library was never loaded by this test
        return
    import weight_only_quantized_fp6_b200 as fp6
    torch.cuda.synchronize()
    status = fp6.device_status()
    assert status == 0, f"device error word set after {request.node.nodeid}: {status}"
