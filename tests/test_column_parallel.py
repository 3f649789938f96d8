"""The column-parallel split of one layer across ranks (host logic, on CPU).

What runs on each rank's GPU is the same fp6_linear call the other tests
check; what is specific to the split is host logic: which rows a rank owns,
where they sit in the packed buffer, and how the ranks' output columns are
gathered back.  These tests pin that logic against the oracle, and run the
gather as two gloo ranks on the CPU, with the oracle standing in for each
rank's GPU call.
"""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from weight_only_quantized_fp6_b200 import column_parallel as cp  # noqa: E402
from weight_only_quantized_fp6_b200 import inputs  # noqa: E402


@pytest.mark.parametrize("N", [128, 256, 1280, 8192, 10240, 57344])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8, 100])
def test_shard_rows_cover_and_balance(N, world):
    spans = [cp.shard_rows(N, world, r) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == N
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 == b0                                   # contiguous, in rank order
    widths = [b - a for a, b in spans]
    assert all(w % 128 == 0 and w >= 0 for w in widths)
    assert max(widths) - min(widths) <= 128               # whole tiles, as even as possible


def test_shard_rows_rejects_bad_arguments():
    with pytest.raises(ValueError):
        cp.shard_rows(100, 2, 0)
    with pytest.raises(ValueError):
        cp.shard_rows(256, 2, 2)


@pytest.mark.parametrize("world", [2, 3, 4])
def test_packed_slice_is_the_packing_of_the_row_slice(orc, world):
    """The bytes a rank takes from the full packed buffer are exactly what
    packing its own rows alone gives (the oracle's layout, row tiles first)."""
    N, K = 1280, 192
    W = inputs.weights(41, N, K)
    codes, scales = orc.quantize(W)
    packed = orc.prepack(codes)
    for r in range(world):
        p, s, n0, n1 = cp.shard_packed(packed, scales, N, K, world, r)
        assert np.array_equal(p, orc.prepack(codes[n0:n1]))
        assert np.array_equal(s, scales[n0:n1])


@pytest.mark.parametrize("fmt", [0, 1, 2, 3])
def test_packed_slice_other_formats(orc, fmt):
    """The same for the other weight formats: a rank's byte range of the full
    packed buffer is the packing of its rows alone."""
    N, K, world = 640, 128, 3
    ncodes = orc.fpx_codes(fmt)
    codes = np.random.default_rng(fmt).integers(0, ncodes, size=(N, K)).astype(np.uint8)
    packed = orc.fpx_prepack(fmt, codes)
    scales = np.arange(N, dtype=np.uint16)
    for r in range(world):
        p, s, n0, n1 = cp.shard_packed(packed, scales, N, K, world, r, fmt)
        assert np.array_equal(p, orc.fpx_prepack(fmt, codes[n0:n1]))
        assert np.array_equal(s, scales[n0:n1])


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, N, K, M, q, fmt=None):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        _rank_work(rank, world, N, K, M, q, fmt)
    except Exception as e:  # report instead of leaving the parent waiting
        q.put((rank, repr(e)))
        raise
    finally:
        dist.destroy_process_group()


def _rank_work(rank, world, N, K, M, q, fmt=None):
    import oracle
    W = inputs.weights(42, N, K)
    x = inputs.activations(43, M, K)
    if fmt is None:
        codes, scales = oracle.quantize(W)
        packed = oracle.prepack(codes)
    else:
        codes, scales = oracle.fpx_quantize(fmt, W)
        packed = oracle.fpx_prepack(fmt, codes)
    p, s, n0, n1 = cp.shard_packed(packed, scales, N, K, world, rank, fmt)
    # this rank's output columns, from its slice of the packed weight only
    if fmt is None:
        y_local = oracle.linear(x, oracle.unpack(p, n1 - n0, K), s)
    else:
        y_local = oracle.fpx_linear(fmt, x, oracle.fpx_unpack(fmt, p, n1 - n0, K), s)
    y = cp.gather_columns(torch.from_numpy(y_local.view(np.float16)), N)
    q.put((rank, y.numpy().view(np.uint16)))


@pytest.mark.parametrize("world,N", [(2, 1280), (3, 1280), (2, 128)])
def test_gloo_ranks_gather_the_full_output(orc, world, N):
    import torch.multiprocessing as mp
    K, M = 192, 5
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, N, K, M, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    results = dict(q.get(timeout=120) for _ in range(world))
    for pr in procs:
        pr.join(timeout=120)
        assert pr.exitcode == 0
    W = inputs.weights(42, N, K)
    x = inputs.activations(43, M, K)
    codes, scales = orc.quantize(W)
    ref = orc.linear(x, codes, scales)
    for r in range(world):
        assert not isinstance(results[r], str), f"rank {r} failed: {results[r]}"
        assert np.array_equal(results[r], ref), f"rank {r}"


@pytest.mark.parametrize("fmt", [1, 2, 3])
def test_gloo_ranks_gather_other_formats(orc, fmt):
    """Two gloo ranks, each computing its columns from its byte range of a
    packed FP6 e2m3 / FP4 / FP5 weight, gather the full oracle output."""
    import torch.multiprocessing as mp
    world, N, K, M = 2, 384, 192, 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, N, K, M, q, fmt)) for r in range(world)]
    for pr in procs:
        pr.start()
    results = dict(q.get(timeout=120) for _ in range(world))
    for pr in procs:
        pr.join(timeout=120)
        assert pr.exitcode == 0
    W = inputs.weights(42, N, K)
    x = inputs.activations(43, M, K)
    codes, scales = orc.fpx_quantize(fmt, W)
    ref = orc.fpx_linear(fmt, x, codes, scales)
    for r in range(world):
        assert not isinstance(results[r], str), f"rank {r} failed: {results[r]}"
        assert np.array_equal(results[r], ref), f"rank {r}"
