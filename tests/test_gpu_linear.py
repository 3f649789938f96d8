"""GPU fp6_linear against the CPU oracle.

Small shapes are compared element by element over the whole output; the
workload shapes (Llama-70B and OPT-30B linear layers, prefill sizes) are
compared on sampled weight rows (two whole 128-row tiles plus random rows) and,
for M > 32, sampled tokens -- through the same library call the benchmark
times.
"""
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


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def as_f16(bits_np):
    return dev(bits_np.view(np.int16)).view(torch.float16)


def bits16(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def gpu_layer(fp6, W):
    codes, scales = fp6.quantize(dev(W))
    return codes, scales, fp6.prepack(codes)


def run_case(fp6, orc, N, K, M, wseed, xseed, outliers=0.0):
    from weight_only_quantized_fp6_b200 import inputs
    W = inputs.weights(wseed, N, K, outlier_p=outliers)
    x = inputs.activations(xseed, M, K)
    codes, scales, packed = gpu_layer(fp6, W)
    y = fp6.linear(as_f16(x), packed, scales, N, K)
    codes_o, scales_o = orc.quantize(W)
    assert np.array_equal(codes.cpu().numpy(), codes_o)
    ref = orc.linear(x, codes_o, scales_o, nthreads=8)
    parity.assert_close(bits16(y), ref, f"N={N} K={K} M={M}")
    return bits16(y), ref


def test_tiny_config(fp6, orc):
    """Tiny W6A16 case: M=4, N=256, K=512, seed 0."""
    from weight_only_quantized_fp6_b200 import inputs
    run_case(fp6, orc, 256, 512, 4, inputs.weight_seed("tiny", 0), inputs.activation_seed(0, 4))


@pytest.mark.parametrize("M", [1, 2, 3, 5, 15, 16, 17, 31, 33, 64, 65, 100, 128, 129, 256, 300])
def test_ragged_tokens(fp6, orc, M):
    """Token counts that leave ragged tails in every MMA tile width."""
    run_case(fp6, orc, 384, 640, M, 77, 1000 + M)


@pytest.mark.parametrize("N,K", [(128, 64), (128, 128), (256, 64), (1280, 192), (640, 4096), (2048, 1024)])
def test_grid_shapes(fp6, orc, N, K):
    """Fewer iterations than SMs, one tile per CTA, tiles split across CTAs."""
    for M in (1, 16, 40):
        run_case(fp6, orc, N, K, M, N + K, M)


@pytest.mark.parametrize("M,N,K", [(128, 128, 1024), (100, 256, 4096), (300, 128, 8192), (128, 128, 18944),
                                   (65, 384, 8192)])
def test_general_kernel_many_contributors(fp6, orc, M, N, K):
    """The M > 64 kernel with row tiles split over 8 to 148 CTAs: the finish
    at the end of a range draws more partials than a warp has copy buffers,
    CTAs hold a first and a last segment of different tiles, and some tiles
    are finished by a CTA that still has work.  Every output is compared, and
    a second launch must give the same bits (the sum order does not depend
    on which CTA finishes)."""
    from weight_only_quantized_fp6_b200 import inputs
    y, _ = run_case(fp6, orc, N, K, M, 9000 + N + K, 9100 + M)
    W = inputs.weights(9000 + N + K, N, K)
    x = inputs.activations(9100 + M, M, K)
    codes, scales, packed = gpu_layer(fp6, W)
    for _ in range(2):
        assert np.array_equal(bits16(fp6.linear(as_f16(x), packed, scales, N, K)), y)


def test_one_hot_bit_exact(fp6, orc):
    """x = identity rows: y[m,n] = fp16_rne(scale[n] * decode(c[n,m])) exactly."""
    from weight_only_quantized_fp6_b200 import inputs
    N, K = 512, 256
    W = inputs.weights(4242, N, K, outlier_p=0.01)
    codes, scales, packed = gpu_layer(fp6, W)
    for M in (16, 64, 256):
        x = np.zeros((M, K), dtype=np.float16)
        idx = np.arange(M) % K
        x[np.arange(M), idx] = 1.0
        y = bits16(fp6.linear(as_f16(x.view(np.uint16)), packed, scales, N, K))
        codes_o, scales_o = orc.quantize(W)
        ref = orc.linear(x.view(np.uint16), codes_o, scales_o)
        nz = (ref & 0x7FFF) != 0
        assert np.array_equal(y[nz], ref[nz])
        assert not (y[~nz] & 0x7FFF).any()


def test_subnormal_weights_survive(fp6, orc):
    """Rows of e3m2 subnormal codes (fp16 subnormals inside the MMA) with
    one-hot activations: no flush to zero."""
    N, K = 128, 64
    codes = np.full((N, K), 0x01, dtype=np.uint8)
    codes[:, 1::2] = 0x23  # -0.1875
    packed = fp6.prepack(dev(codes))
    scales = dev(np.full(N, 1.0, dtype=np.float16))
    x = np.zeros((16, K), dtype=np.float16)
    x[np.arange(16), np.arange(16)] = 1.0
    y = fp6.linear(as_f16(x.view(np.uint16)), packed, scales, N, K).cpu().float().numpy()
    want = np.where(np.arange(16) % 2 == 0, 0.0625, -0.1875)
    assert np.array_equal(y, np.tile(want[:, None], (1, N)))


def test_zero_activations_and_zero_rows(fp6):
    from weight_only_quantized_fp6_b200 import inputs
    N, K = 256, 512
    W = inputs.weights(3, N, K)
    W[7] = 0.0
    codes, scales, packed = gpu_layer(fp6, W)
    y = fp6.linear(torch.zeros((9, K), dtype=torch.float16, device="cuda"), packed, scales, N, K)
    assert not (bits16(y) & 0x7FFF).any()
    x = torch.randn(9, K, device="cuda").half()
    y = fp6.linear(x, packed, scales, N, K)
    assert not (bits16(y)[:, 7] & 0x7FFF).any()


def test_k_zero_and_m_zero(fp6):
    packed = torch.zeros(16, dtype=torch.uint8, device="cuda")
    scales = torch.ones(128, dtype=torch.float16, device="cuda")
    y = torch.full((3, 128), 5.0, dtype=torch.float16, device="cuda")
    fp6.linear(torch.zeros((3, 0), dtype=torch.float16, device="cuda"), packed, scales, 128, 0, out=y)
    assert (y == 0).all()
    y0 = fp6.linear(torch.zeros((0, 64), dtype=torch.float16, device="cuda"),
                    torch.zeros(6144, dtype=torch.uint8, device="cuda"), scales, 128, 64)
    assert y0.shape == (0, 128)


def test_deterministic(fp6):
    from weight_only_quantized_fp6_b200 import inputs
    N, K = 1024, 4096
    codes, scales, packed = gpu_layer(fp6, inputs.weights(9, N, K))
    for M in (1, 16, 200):
        x = torch.randn(M, K, device="cuda").half()
        a = bits16(fp6.linear(x, packed, scales, N, K))
        b = bits16(fp6.linear(x, packed, scales, N, K))
        assert np.array_equal(a, b)


def test_errors_are_reported(fp6):
    N, K = 256, 512
    scales = torch.ones(N, dtype=torch.float16, device="cuda")
    packed = torch.zeros(N * K * 3 // 4, dtype=torch.uint8, device="cuda")
    xbuf = torch.zeros((4 * K + 8,), dtype=torch.float16, device="cuda")
    x_mis = xbuf[1:1 + 4 * K].view(4, K)  # 2-byte offset: misaligned
    with pytest.raises(fp6.FP6Error) as e:
        fp6.linear(x_mis, packed, scales, N, K)
    assert e.value.status == 3
    from weight_only_quantized_fp6_b200 import _lib
    lib = _lib.load()
    x = torch.zeros((4, K), dtype=torch.float16, device="cuda")
    y = torch.empty((4, N), dtype=torch.float16, device="cuda")
    need = fp6.workspace_bytes(4, N, K)
    assert need > 0
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    st = lib.fp6_linear(x.data_ptr(), packed.data_ptr(), scales.data_ptr(), 4, N, K, y.data_ptr(),
                        ws.data_ptr(), need - 16, None)
    assert st == 6
    st = lib.fp6_linear(x.data_ptr(), packed.data_ptr(), scales.data_ptr(), 4, N, K, y.data_ptr(),
                        None, 0, None)
    assert st == 6


def test_no_device_errors_recorded(fp6):
    torch.cuda.synchronize()
    assert fp6.device_status() == 0


# ---- the workload shapes, sampled ------------------------------------------------

WORKLOADS = []
for wname in ("llama70b_o_decode", "llama70b_all", "opt30b", "prefill"):
    spec = __import__("weight_only_quantized_fp6_b200.inputs", fromlist=["WORKLOADS"]).WORKLOADS[wname]
    for li, (lname, (N, K)) in enumerate(spec["layers"].items()):
        WORKLOADS.append(pytest.param(wname, li, lname, N, K, spec["M"], spec["outliers"],
                                      id=f"{wname}-{lname}"))


@pytest.mark.parametrize("wname,li,lname,N,K,Ms,outliers", WORKLOADS)
def test_workload_sampled(fp6, orc, wname, li, lname, N, K, Ms, outliers):
    from weight_only_quantized_fp6_b200 import inputs
    wseed = inputs.weight_seed(wname, li)
    W = parity.gen_weights_parallel(wseed, N, K, outliers)
    codes, scales, packed = gpu_layer(fp6, W)
    del W
    rng = np.random.default_rng(wseed)
    rows = parity.sample_rows(N, rng)
    W_rows = inputs.weights(wseed, N, K, rows=rows, outlier_p=outliers)
    codes_o, scales_o = orc.quantize(W_rows)
    rows_t = torch.from_numpy(rows).cuda()
    assert np.array_equal(codes.index_select(0, rows_t).cpu().numpy(), codes_o)
    assert np.array_equal(bits16(scales.index_select(0, rows_t)), scales_o)
    # the first row tile's packed bytes, byte for byte
    tile_bytes = (K // 64) * 6144
    assert np.array_equal(packed[:tile_bytes].cpu().numpy(), orc.prepack(codes_o[:128]))
    for M in Ms:
        x = inputs.activations(inputs.activation_seed(wseed, M), M, K)
        y = bits16(fp6.linear(as_f16(x), packed, scales, N, K))
        toks = parity.sample_tokens(M, rng)
        ref = orc.linear(x[toks], codes_o, scales_o, nthreads=16)
        parity.assert_close(y[np.ix_(toks, rows)], ref, f"{lname} N={N} K={K} M={M}")


@pytest.mark.parametrize("N,K,M", [(18944, 128, 300), (18944, 128, 1100), (148 * 128 * 2, 192, 257)])
def test_wave_schedule(fp6, orc, N, K, M):
    """Shapes whose tiles fill whole waves of 148 CTAs (148 or 296 row tiles
    times 2 or 5 token tiles, the last token tile ragged), through the general
    kernel; checked on sampled rows (two whole 128-row tiles and random rows)
    and sampled tokens."""
    from weight_only_quantized_fp6_b200 import inputs
    W = inputs.weights(N + K, N, K)
    x = inputs.activations(M, M, K)
    codes, scales, packed = gpu_layer(fp6, W)
    y = bits16(fp6.linear(as_f16(x), packed, scales, N, K))
    rng = np.random.default_rng(N + M)
    rows = parity.sample_rows(N, rng)
    toks = parity.sample_tokens(M, rng, limit=48)
    codes_o, scales_o = orc.quantize(W[rows])
    ref = orc.linear(x[toks], codes_o, scales_o, nthreads=16)
    parity.assert_close(y[np.ix_(toks, rows)], ref, f"wave N={N} K={K} M={M}")


def test_workspace_reused_across_shapes(fp6, orc):
    """One workspace serves a sequence of problems of different sizes: the
    counters left by each call (and the partials it wrote) never disturb the
    next call."""
    from weight_only_quantized_fp6_b200 import inputs
    ws = fp6.Workspace(torch.device("cuda"))
    for (N, K, M) in [(256, 512, 3), (1280, 4096, 1), (384, 640, 17), (2560, 2048, 8), (128, 64, 2),
                      (1280, 4096, 1), (640, 8192, 40)]:
        W = inputs.weights(N * 7 + K, N, K)
        x = inputs.activations(M + N, M, K)
        codes, scales, packed = gpu_layer(fp6, W)
        y = fp6.linear(as_f16(x), packed, scales, N, K, workspace=ws)
        codes_o, scales_o = orc.quantize(W)
        parity.assert_close(bits16(y), orc.linear(x, codes_o, scales_o, nthreads=8), f"N={N} K={K} M={M}")


@pytest.fixture(scope="module")
def split_heavy_layer(orc):
    N, K = 21504, 7168
    W = parity.gen_weights_parallel(4242, N, K, 0.0)
    codes_o, scales_o = orc.quantize(W)
    return W, codes_o, scales_o


@pytest.mark.parametrize("M", [1, 16, 32])
def test_split_heavy_layer_every_row(fp6, orc, split_heavy_layer, M):
    """OPT-30B QKV shape (N = 21504, K = 7168): every persistent CTA covers
    more than one row tile, so ranges hold up to three segments and every
    split tile is finished by another CTA than the ones that published its
    partials.  The whole output is compared, not a sample, so a row tile whose
    fix-up went wrong cannot hide."""
    from weight_only_quantized_fp6_b200 import inputs
    N, K = 21504, 7168
    W, codes_o, scales_o = split_heavy_layer
    codes, scales, packed = gpu_layer(fp6, W)
    x = inputs.activations(4243 + M, M, K)
    y = bits16(fp6.linear(as_f16(x), packed, scales, N, K))
    assert np.array_equal(codes.cpu().numpy(), codes_o)
    ref = orc.linear(x, codes_o, scales_o, nthreads=16)
    parity.assert_close(y, ref, f"N={N} K={K} M={M}")
