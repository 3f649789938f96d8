"""GPU s24_* entry points (2:4 structured-sparse INT4 weights, the
Sparse-Marlin format) against the oracle.

Quantize (kept positions, codes, scales) and prepack are compared byte for
byte, including rows of pruning ties and rounding ties; dequant is compared
bit for bit with every code value and every position pair at every tile
position; the linear layer is compared with the tolerance of the e3m2 tests
over whole small outputs (every kernel variant), on sampled rows and tokens of
the Llama-70B O-projection shape, and bit for bit with one-hot activations.
"""
import numpy as np
import pytest

from tests import parity

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

S24 = 4
PAIRS = [(0, 1), (0, 2), (0, 3), (1, 2), (1, 3), (2, 3)]


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


def as_f16(bits_np):
    return dev(bits_np.view(np.int16)).view(torch.float16)


def host(t):
    return t.cpu().numpy()


def bits16(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def check_quantize(fp6, orc, W):
    q_g, pos_g, s_g = fp6.s24_quantize(dev(W))
    q_o, pos_o, s_o = orc.s24_quantize(W)
    assert np.array_equal(bits16(s_g), s_o)
    assert np.array_equal(host(pos_g), pos_o)
    assert np.array_equal(host(q_g), q_o)
    packed = fp6.s24_prepack(q_g, pos_g)
    assert np.array_equal(host(packed), orc.s24_prepack(q_o, pos_o))
    return q_o, pos_o, s_o, packed


@pytest.mark.parametrize("N,K,seed,outliers", [(256, 512, 0, 0.0), (384, 1280, 1, 0.001)])
def test_quantize_prepack_match_oracle(fp6, orc, N, K, seed, outliers):
    from weight_only_quantized_fp6_b200 import inputs
    check_quantize(fp6, orc, inputs.weights(seed, N, K, outlier_p=outliers))


def test_quantize_ties(fp6, orc):
    """Rows whose scale is exactly s0 (largest magnitude 7*s0): every rounding
    midpoint (m + 1/2)*s0 below 7*s0 and the floats beside it, both signs, and
    groups with equal magnitudes (pruning ties), zeros and -0."""
    N, K = 128, 256
    rng = np.random.default_rng(24)
    W = np.zeros((N, K), dtype=np.float32)
    for n in range(N):
        s0 = np.float32(2.0 ** int(rng.integers(-12, 4)) * (1 + int(rng.integers(0, 1024)) / 1024))
        vals = []
        for m in range(7):
            t = np.float32((m + 0.5) * s0)
            vals += [t, np.nextafter(t, np.float32(0)), np.nextafter(t, np.float32(np.inf))]
        vals = np.array(vals, dtype=np.float32)
        vals *= np.where(rng.random(vals.size) < 0.5, -1.0, 1.0).astype(np.float32)
        row = np.resize(vals, K)
        # pruning ties: groups of four equal magnitudes, pairs of equal maxima
        row[0:4] = s0
        row[4:8] = [-s0, s0, -s0, s0]
        row[8:12] = [0.0, -0.0, 0.0, -0.0]
        row[12:16] = [2 * s0, 3 * s0, 3 * s0, 2 * s0]
        row[16:20] = [6.5 * s0, -6.5 * s0, 5.5 * s0, -4.5 * s0]
        row[20] = np.float32(7 * s0)                       # sets the scale to exactly s0
        W[n] = row
    W[5] = 0.0                                             # a row of zeros
    check_quantize(fp6, orc, W)


def test_every_code_and_position_pair(fp6, orc):
    """Every code value and every kept-position pair at every group of a tile,
    through prepack and dequant (with and without scales)."""
    N, K = 256, 128
    rows = np.arange(N)[:, None]
    groups = np.arange(K // 4)[None, :]
    q = np.zeros((N, K // 2), dtype=np.int8)
    pos = np.zeros((N, K // 2), dtype=np.uint8)
    pair = (rows * 7 + groups * 5) % 6
    q[:, 0::2] = ((rows * 3 + groups) % 16) - 8
    q[:, 1::2] = ((rows + groups * 11) % 16) - 8
    for p, (i0, i1) in enumerate(PAIRS):
        pos[:, 0::2][pair == p] = i0
        pos[:, 1::2][pair == p] = i1
    packed = fp6.s24_prepack(dev(q), dev(pos))
    packed_o = orc.s24_prepack(q, pos)
    assert np.array_equal(host(packed), packed_o)
    assert np.array_equal(bits16(fp6.dequant(packed, None, N, K, fmt=S24)), orc.s24_dequant(packed_o, None, N, K))
    scales = (2.0 ** np.random.default_rng(3).uniform(-14, 8, N)).astype(np.float16)
    got = fp6.dequant(packed, dev(scales), N, K, fmt=S24)
    assert np.array_equal(bits16(got), orc.s24_dequant(packed_o, scales.view(np.uint16), N, K))


def run_linear(fp6, orc, N, K, M, wseed, xseed, outliers=0.0):
    from weight_only_quantized_fp6_b200 import inputs
    W = inputs.weights(wseed, N, K, outlier_p=outliers)
    x = inputs.activations(xseed, M, K)
    layer = fp6.FP6Linear.from_float(dev(W), fmt=S24)
    y = layer(as_f16(x))
    q_o, pos_o, s_o = orc.s24_quantize(W)
    assert np.array_equal(host(layer.packed), orc.s24_prepack(q_o, pos_o))
    ref = orc.s24_linear(x, q_o, pos_o, s_o)
    parity.assert_close(bits16(y), ref, f"s24 N={N} K={K} M={M}")


@pytest.mark.parametrize("M", [1, 5, 16, 17, 33, 64, 65, 129, 300])
def test_linear_ragged_tokens(fp6, orc, M):
    """Every kernel variant (16 / 32 / 64 token columns, 128 / 256) with ragged tails."""
    run_linear(fp6, orc, 384, 640, M, 77, 1000 + M)


@pytest.mark.parametrize("N,K", [(128, 64), (256, 64), (1280, 192), (640, 4096)])
def test_linear_grid_shapes(fp6, orc, N, K):
    for M in (1, 40):
        run_linear(fp6, orc, N, K, M, N + K, M)


def test_one_hot_bit_exact(fp6, orc):
    """x = identity rows: y[m,n] = fp16_rne(scale[n] * v[n,m]), exactly the
    oracle's dense dequantized weight."""
    from weight_only_quantized_fp6_b200 import inputs
    N, K = 256, 128
    layer = fp6.FP6Linear.from_float(dev(inputs.weights(5, N, K)), fmt=S24)
    W16 = orc.s24_dequant(host(layer.packed), bits16(layer.scales), N, K)
    for M in (16, 64, 128):
        x = np.zeros((M, K), dtype=np.float16)
        x[np.arange(M), np.arange(M) % K] = 1.0
        y = layer(dev(x))
        assert np.array_equal(parity.f16(bits16(y)), parity.f16(W16[:, np.arange(M) % K].T))


@pytest.mark.parametrize("M", [1, 16, 64, 1024])
def test_llama70b_o_proj_sampled(fp6, orc, M):
    """N = K = 8192 in the benchmark's launch configuration, on sampled weight
    rows (two whole tiles and random rows) and tokens."""
    from weight_only_quantized_fp6_b200 import inputs
    N = K = 8192
    rng = np.random.default_rng(200 + M)
    W = inputs.weights_parallel(11, N, K, 0.0)
    x = inputs.activations(12, M, K)
    layer = fp6.FP6Linear.from_float(dev(W), fmt=S24)
    y = layer(as_f16(x))
    rows = parity.sample_rows(N, rng)
    toks = parity.sample_tokens(M, rng)
    q_o, pos_o, s_o = orc.s24_quantize(W[rows])
    assert np.array_equal(bits16(layer.scales)[rows], s_o)
    ref = orc.s24_linear(x[toks], q_o, pos_o, s_o)
    parity.assert_close(bits16(y)[np.ix_(toks, rows)], ref, f"s24 M={M}")


def test_errors(fp6):
    from weight_only_quantized_fp6_b200 import _lib
    lib = _lib.load()
    W = torch.zeros((128, 66), dtype=torch.float32, device="cuda")
    q = torch.empty((128, 33), dtype=torch.int8, device="cuda")
    pos = torch.empty((128, 33), dtype=torch.uint8, device="cuda")
    s = torch.empty(128, dtype=torch.float16, device="cuda")
    assert lib.s24_quantize(W.data_ptr(), 128, 66, q.data_ptr(), pos.data_ptr(), s.data_ptr(), None) == 2
    W = torch.full((128, 64), float("nan"), dtype=torch.float32, device="cuda")
    with pytest.raises(fp6.FP6Error) as e:
        fp6.s24_quantize(W)
    assert e.value.status == 4
    assert lib.s24_packed_bytes(100, 64) == 0
    assert lib.s24_packed_bytes(128, 64) == 128 * 64 * 3 // 8
