"""Column-parallel FP6 linear layer over several GPUs (one process per GPU).

The output features N are split across ranks in whole 128-row weight tiles:
rank r owns rows [n0, n1) of W, i.e. one contiguous byte range of the packed
buffer (tiles are stored row-tile major) and the matching scales.  Every rank
receives the full activations x and computes its own block of output columns
y[:, n0:n1] with fp6_linear on its GPU; no data crosses GPUs unless the caller
asks for the full y, which one all-gather over the process group assembles.

This is the split the FP6-LLM pages point to when they compare one GPU running
FP6 with two GPUs running FP16: the weights are divided, the activations are
not.  The split itself and the gather are plain host logic and collectives;
every step of the product runs in libfp6.
"""
from __future__ import annotations

from fractions import Fraction

from . import _lib

TILE_ROWS = 128

# bytes per weight of each packed format (None = FP6 e3m2, as fp6_*)
_BYTES_PER_WEIGHT = {None: Fraction(3, 4), 0: Fraction(3, 4), 1: Fraction(3, 4), 2: Fraction(1, 2),
                     3: Fraction(5, 8), 4: Fraction(3, 8)}


def shard_rows(N: int, world: int, rank: int) -> tuple[int, int]:
    """Rows [n0, n1) of an N-row weight owned by `rank`: whole 128-row tiles,
    split as evenly as possible (the first N/128 mod world ranks get one
    tile more).  A rank may own no rows when there are fewer tiles than ranks."""
    if N % TILE_ROWS != 0:
        raise ValueError("N must be a multiple of 128")
    if not (0 <= rank < world):
        raise ValueError("rank out of range")
    tiles = N // TILE_ROWS
    t0 = rank * tiles // world
    t1 = (rank + 1) * tiles // world
    return t0 * TILE_ROWS, t1 * TILE_ROWS


def packed_range(K: int, n0: int, n1: int, fmt=None) -> tuple[int, int]:
    """Byte range [b0, b1) of rows [n0, n1) inside the packed buffer of an
    N x K weight: every format stores its 128-row tiles one after another, so
    whole row tiles are one contiguous range (0.75 bytes per weight for the
    6-bit formats, 0.625 for FP5, 0.5 for FP4, 0.375 for 2:4 sparse INT4)."""
    if n0 % TILE_ROWS or n1 % TILE_ROWS or K % 64:
        raise ValueError("rows must be whole 128-row tiles and K a multiple of 64")
    if fmt not in _BYTES_PER_WEIGHT:
        raise ValueError(f"unknown format {fmt!r}")
    b = _BYTES_PER_WEIGHT[fmt]
    return int(n0 * K * b), int(n1 * K * b)


def shard_packed(packed, scales, N: int, K: int, world: int, rank: int, fmt=None):
    """This rank's (packed, scales, n0, n1) views of a full packed weight."""
    n0, n1 = shard_rows(N, world, rank)
    b0, b1 = packed_range(K, n0, n1, fmt)
    return packed[b0:b1], scales[n0:n1], n0, n1


def gather_columns(y_local, N: int, group=None):
    """Assemble y[M, N] on every rank from the ranks' column blocks
    y_local[M, n1 - n0] (in rank order), with one all-gather.  Blocks of
    unequal width are padded to the widest for the collective."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    M = y_local.shape[0]
    widths = [shard_rows(N, world, r)[1] - shard_rows(N, world, r)[0] for r in range(world)]
    wmax = max(widths)
    send = torch.zeros((wmax, M), dtype=y_local.dtype, device=y_local.device)
    send[: y_local.shape[1]] = y_local.t()
    recv = torch.empty((world * wmax, M), dtype=y_local.dtype, device=y_local.device)
    dist.all_gather_into_tensor(recv, send, group=group)
    blocks = [recv[r * wmax: r * wmax + widths[r]] for r in range(world)]
    return torch.cat(blocks, dim=0).t().contiguous()


class ColumnParallelFP6Linear:
    """y = x . (scale (.) decode(W))^T with W's rows split across the ranks of
    `group` (torch.distributed, NCCL on GPUs); `fmt` selects the weight format
    as in linear().  Construct it on every rank
    from the full packed weight (only this rank's slice is kept on its GPU) or
    from an already sliced one (pass shard=True)."""

    def __init__(self, packed, scales, N: int, K: int, group=None, shard: bool = False, fmt=None):
        import torch.distributed as dist
        self.group = group
        self.fmt = fmt
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.N, self.K = N, K
        self.n0, self.n1 = shard_rows(N, self.world, self.rank)
        if shard:
            self.packed, self.scales = packed, scales
        else:
            self.packed, self.scales, _, _ = shard_packed(packed, scales, N, K, self.world, self.rank, fmt)
            self.packed = self.packed.contiguous().clone()
            self.scales = self.scales.contiguous().clone()

    def local(self, x, out=None):
        """This rank's output columns y[:, n0:n1]."""
        from . import linear
        _lib.load()                          # fail loudly without the CUDA library
        return linear(x, self.packed, self.scales, self.n1 - self.n0, self.K, out=out, fmt=self.fmt)

    def __call__(self, x, gather: bool = True):
        y = self.local(x)
        return gather_columns(y, self.N, self.group) if gather else y
