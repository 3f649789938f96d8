"""GPU fpx_* entry points (FP6 e2m3, FP4 e2m1, FP5 e2m2, and e3m2 through
the same calls) against the oracle.

Quantize, prepack and dequant are compared byte for byte, with every code at
every position of a tile (which also fixes which nibble of a byte the FP4
conversion reads first, and the FP5 rebuild's bit gathering); the linear layer is compared with the tolerance of
the e3m2 tests, over whole small outputs and on sampled rows and tokens of the
Llama-70B O-projection shape.
"""
import numpy as np
import pytest

from tests import parity

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

FORMATS = [0, 1, 2, 3]       # e3m2, e2m3, e2m1, e2m2
NAMES = {0: "e3m2", 1: "e2m3", 2: "e2m1", 3: "e2m2"}


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


@pytest.mark.parametrize("fmt", FORMATS)
def test_every_code_at_every_tile_position(fp6, orc, fmt):
    ncodes = orc.fpx_codes(fmt)
    N, K = 256, 128
    rows = np.arange(N)[:, None]
    cols = np.arange(K)[None, :]
    codes = ((rows * 5 + cols * 3 + (rows // 64)) % ncodes).astype(np.uint8)
    codes[:ncodes] = (np.arange(ncodes)[:, None] + cols) % ncodes   # each code in each column
    packed_g = fp6.prepack(dev(codes), fmt=fmt)
    packed_o = orc.fpx_prepack(fmt, codes)
    assert np.array_equal(host(packed_g), packed_o)
    plain = fp6.dequant(packed_g, None, N, K, fmt=fmt)
    assert np.array_equal(bits16(plain), orc.fpx_dequant(fmt, packed_o, None, N, K))
    scales = (2.0 ** np.random.default_rng(fmt).uniform(-14, 8, N)).astype(np.float16)
    scaled = fp6.dequant(packed_g, dev(scales), N, K, fmt=fmt)
    assert np.array_equal(bits16(scaled), orc.fpx_dequant(fmt, packed_o, scales.view(np.uint16), N, K))


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("N,K,seed,outliers", [(256, 512, 0, 0.0), (384, 1280, 1, 0.001)])
def test_quantize_prepack_match_oracle(fp6, orc, fmt, N, K, seed, outliers):
    from weight_only_quantized_fp6_b200 import inputs
    W = inputs.weights(seed, N, K, outlier_p=outliers)
    codes_g, scales_g = fp6.quantize(dev(W), fmt=fmt)
    codes_o, scales_o = orc.fpx_quantize(fmt, W)
    assert np.array_equal(bits16(scales_g), scales_o)
    assert np.array_equal(host(codes_g), codes_o)
    assert np.array_equal(host(fp6.prepack(codes_g, fmt=fmt)), orc.fpx_prepack(fmt, codes_o))


@pytest.mark.parametrize("fmt", FORMATS)
def test_quantize_ties_and_neighbours(fp6, orc, fmt):
    """Rows whose scale is a power of two (largest magnitude x 2^e): every
    midpoint between neighbouring magnitudes (a tie), the floats on either
    side of it, and values beyond the largest magnitude, with both signs."""
    table = orc.fpx_decode_table(fmt)
    mags = table[: len(table) // 2]
    top = mags[-1]
    mids = (mags[:-1] + mags[1:]) / 2
    N, K = 128, 64 * 4
    W = np.zeros((N, K), dtype=np.float32)
    rng = np.random.default_rng(10 + fmt)
    for n in range(N):
        e = int(rng.integers(-10, 6))
        s = 2.0 ** e
        vals = [top * s]                                            # sets the scale to exactly 2^e
        for m in mids:
            t = np.float32(m * s)
            vals += [t, np.nextafter(t, np.float32(0)), np.nextafter(t, np.float32(np.inf))]
        vals += [top * s * 0.999, 0.0, -0.0]
        vals = np.array(vals, dtype=np.float32)
        sign = np.where(rng.random(vals.size) < 0.5, -1.0, 1.0).astype(np.float32)
        vals = vals * sign
        vals[0] = top * s
        row = np.resize(vals, K)
        W[n] = row
    codes_g, scales_g = fp6.quantize(dev(W), fmt=fmt)
    codes_o, scales_o = orc.fpx_quantize(fmt, W)
    assert np.array_equal(bits16(scales_g), scales_o)
    assert np.array_equal(host(codes_g), codes_o)


def run_linear(fp6, orc, fmt, N, K, M, wseed, xseed, outliers=0.0):
    from weight_only_quantized_fp6_b200 import inputs
    W = inputs.weights(wseed, N, K, outlier_p=outliers)
    x = inputs.activations(xseed, M, K)
    codes, scales = fp6.quantize(dev(W), fmt=fmt)
    packed = fp6.prepack(codes, fmt=fmt)
    y = fp6.linear(as_f16(x), packed, scales, N, K, fmt=fmt)
    codes_o, scales_o = orc.fpx_quantize(fmt, W)
    assert np.array_equal(host(codes), codes_o)
    ref = orc.fpx_linear(fmt, x, codes_o, scales_o)
    parity.assert_close(bits16(y), ref, f"{NAMES[fmt]} N={N} K={K} M={M}")
    return y, packed, scales


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("M", [1, 5, 16, 17, 33, 64, 65, 129, 300])
def test_linear_ragged_tokens(fp6, orc, fmt, M):
    """Every kernel variant (16 / 32 / 64 token columns, 128 / 256) with ragged tails."""
    run_linear(fp6, orc, fmt, 384, 640, M, 77, 1000 + M)


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("N,K", [(128, 64), (256, 64), (1280, 192), (640, 4096)])
def test_linear_grid_shapes(fp6, orc, fmt, N, K):
    for M in (1, 40):
        run_linear(fp6, orc, fmt, N, K, M, N + K, M)


@pytest.mark.parametrize("fmt", [1, 2, 3])
def test_one_hot_bit_exact(fp6, orc, fmt):
    """x = identity rows: y[m,n] = fp16_rne(scale[n] * decode(c[n,m])), exactly
    the oracle's dequantized weight."""
    from weight_only_quantized_fp6_b200 import inputs
    N, K = 256, 128
    W = inputs.weights(5, N, K)
    codes, scales = fp6.quantize(dev(W), fmt=fmt)
    packed = fp6.prepack(codes, fmt=fmt)
    for M in (16, 64, 128):
        x = np.zeros((M, K), dtype=np.float16)
        x[np.arange(M), np.arange(M) % K] = 1.0
        y = fp6.linear(dev(x), packed, scales, N, K, fmt=fmt)
        W16 = orc.fpx_dequant(fmt, host(packed), bits16(scales), N, K)
        # compared as values: a -0 weight comes out +0 after the fp32 sum with +0 terms
        assert np.array_equal(parity.f16(bits16(y)), parity.f16(W16[:, np.arange(M) % K].T))


def test_e3m2_through_fpx_is_the_fp6_path(fp6):
    """fpx_* with e3m2 gives the same bytes and bits as the fp6_* entry points."""
    from weight_only_quantized_fp6_b200 import inputs
    N, K = 512, 1024
    W = dev(inputs.weights(3, N, K))
    c0, s0 = fp6.quantize(W)
    c1, s1 = fp6.quantize(W, fmt=0)
    assert torch.equal(c0, c1) and torch.equal(s0, s1)
    p0, p1 = fp6.prepack(c0), fp6.prepack(c1, fmt=0)
    assert torch.equal(p0, p1)
    for M in (1, 48, 200):
        x = as_f16(inputs.activations(4, M, K))
        assert torch.equal(fp6.linear(x, p0, s0, N, K), fp6.linear(x, p1, s1, N, K, fmt=0))


@pytest.mark.parametrize("fmt", [1, 2, 3])
@pytest.mark.parametrize("M", [1, 16, 64, 1024])
def test_llama70b_o_proj_sampled(fp6, orc, fmt, M):
    """N = K = 8192 in the launch configuration of the benchmark, on sampled
    weight rows (two whole tiles and random rows) and tokens."""
    from weight_only_quantized_fp6_b200 import inputs
    N = K = 8192
    rng = np.random.default_rng(100 + M + fmt)
    W = inputs.weights_parallel(11, N, K, 0.0)
    x = inputs.activations(12, M, K)
    codes, scales = fp6.quantize(dev(W), fmt=fmt)
    packed = fp6.prepack(codes, fmt=fmt)
    y = fp6.linear(as_f16(x), packed, scales, N, K, fmt=fmt)
    rows = parity.sample_rows(N, rng)
    toks = parity.sample_tokens(M, rng)
    codes_o, scales_o = orc.fpx_quantize(fmt, W[rows])
    assert np.array_equal(host(codes)[rows], codes_o)
    ref = orc.fpx_linear(fmt, x[toks], codes_o, scales_o)
    parity.assert_close(bits16(y)[np.ix_(toks, rows)], ref, f"{NAMES[fmt]} M={M}")
