"""Stored layers on the GPU: FP6Linear.save / load round trip for every
format (the loaded layer gives the same bits as the saved one), and a blob
whose header names another layout version is refused."""
import numpy as np
import pytest

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


@pytest.mark.parametrize("fmt", [None, 1, 2, 3, 4])
def test_save_load_round_trip(fp6, tmp_path, fmt):
    from weight_only_quantized_fp6_b200 import inputs
    N, K = 384, 640
    layer = fp6.FP6Linear.from_float(torch.from_numpy(inputs.weights(31, N, K)).cuda(), fmt=fmt)
    path = tmp_path / "layer.fp6w"
    layer.save(path)
    assert path.stat().st_size == 64 + 2 * N + fp6.packed_bytes(N, K, fmt)
    back = fp6.FP6Linear.load(path)
    assert (back.N, back.K, back.fmt) == (N, K, fmt)
    assert torch.equal(back.packed, layer.packed)
    assert torch.equal(back.scales.view(torch.int16), layer.scales.view(torch.int16))
    x = torch.from_numpy(inputs.activations(32, 17, K).view(np.int16)).cuda().view(torch.float16)
    assert torch.equal(back(x).view(torch.int16), layer(x).view(torch.int16))


def test_other_layout_version_is_refused(fp6, tmp_path):
    from weight_only_quantized_fp6_b200 import inputs
    N, K = 128, 256
    layer = fp6.FP6Linear.from_float(torch.from_numpy(inputs.weights(33, N, K)).cuda())
    path = tmp_path / "layer.fp6w"
    layer.save(path)
    raw = bytearray(path.read_bytes())
    raw[4:8] = (1).to_bytes(4, "little")       # a blob from the first packed layout
    path.write_bytes(bytes(raw))
    with pytest.raises(fp6.FP6Error) as e:
        fp6.FP6Linear.load(path)
    assert e.value.status == 7
