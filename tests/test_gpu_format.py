"""GPU quantize / prepack / dequant against the oracle, byte for byte."""
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


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.cpu().numpy()


def bits16(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def test_all_64_codes_at_every_tile_position(fp6, orc):
    """Exhaustive decode: every code at every (row, column) position of a tile."""
    N, K = 256, 128
    rows = np.arange(N)[:, None]
    cols = np.arange(K)[None, :]
    codes = ((rows * 5 + cols * 3 + (rows // 64)) % 64).astype(np.uint8)
    codes[:64] = (np.arange(64)[:, None] + cols) % 64  # each code at each column too
    packed_g = fp6.prepack(dev(codes))
    packed_o = orc.prepack(codes)
    assert np.array_equal(host(packed_g), packed_o)
    w_plain = fp6.dequant(packed_g, None, N, K)
    assert np.array_equal(bits16(w_plain), orc.dequant(packed_o, None, N, K))
    scales = (2.0 ** np.random.default_rng(0).uniform(-14, 8, N)).astype(np.float16)
    w_sc = fp6.dequant(packed_g, dev(scales), N, K)
    assert np.array_equal(bits16(w_sc), orc.dequant(packed_o, scales.view(np.uint16), N, K))


@pytest.mark.parametrize("N,K,seed,outliers", [(256, 512, 0, 0.0), (384, 1280, 1, 0.001), (128, 64, 2, 0.0)])
def test_quantize_prepack_match_oracle(fp6, orc, N, K, seed, outliers):
    from weight_only_quantized_fp6_b200 import inputs
    W = inputs.weights(seed, N, K, outlier_p=outliers)
    codes_g, scales_g = fp6.quantize(dev(W))
    codes_o, scales_o = orc.quantize(W)
    assert np.array_equal(bits16(scales_g), scales_o)
    assert np.array_equal(host(codes_g), codes_o)
    assert np.array_equal(host(fp6.prepack(codes_g)), orc.prepack(codes_o))


def test_quantize_rounding_edges(fp6, orc):
    """Weights placed exactly on every midpoint and its fp32 neighbours, in
    rows with different scales, plus zero rows and signed zeros."""
    from tests.test_oracle_decode import closed_form
    mags = [float(closed_form(c)) for c in range(32)]
    mids = [(mags[i] + mags[i + 1]) / 2 for i in range(31)]
    K = 256
    rows = []
    for s in (1.0, 0.015625, 0.0009765625, 3.0517578125e-05, 7.5):
        vals = []
        for m in mids:
            v = np.float32(m * s)
            vals += [v, np.nextafter(v, np.float32(0)), np.nextafter(v, np.float32(1e9))]
        vals = [np.float32(28 * s)] + vals
        vals += [-v for v in vals]
        row = np.zeros(K, dtype=np.float32)
        row[:len(vals)] = vals[:K]
        rows.append(row)
    rows.append(np.zeros(K, dtype=np.float32))
    neg0 = np.zeros(K, dtype=np.float32)
    neg0[1:] = -0.0
    neg0[0] = 1.0
    rows.append(neg0)
    W = np.stack(rows + [rows[0]] * (128 - len(rows)))
    codes_g, scales_g = fp6.quantize(dev(W))
    codes_o, scales_o = orc.quantize(W)
    assert np.array_equal(bits16(scales_g), scales_o)
    assert np.array_equal(host(codes_g), codes_o)


def test_quantize_errors(fp6):
    W = np.ones((128, 64), dtype=np.float32)
    W[5, 7] = np.nan
    with pytest.raises(fp6.FP6Error) as e:
        fp6.quantize(dev(W))
    assert e.value.status == 4
    W = np.ones((128, 64), dtype=np.float32)
    W[9, 0] = 3e6
    with pytest.raises(fp6.FP6Error) as e:
        fp6.quantize(dev(W))
    assert e.value.status == 5
    W = np.ones((128, 64), dtype=np.float32)
    codes, scales = fp6.quantize(dev(W))  # and a clean call afterwards succeeds
    assert (host(codes) == 0x1F).all()


def test_prepack_dequant_large_random(fp6, orc):
    rng = np.random.default_rng(7)
    N, K = 1024, 2048
    codes = rng.integers(0, 256, size=(N, K), dtype=np.uint8)  # bits 7..6 must be ignored
    packed_g = fp6.prepack(dev(codes))
    packed_o = orc.prepack(codes & 0x3F)
    assert np.array_equal(host(packed_g), packed_o)
    scales = (2.0 ** rng.uniform(-10, 4, N)).astype(np.float16)
    w = fp6.dequant(packed_g, dev(scales), N, K)
    assert np.array_equal(bits16(w), orc.dequant(packed_o, scales.view(np.uint16), N, K))
