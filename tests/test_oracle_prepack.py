"""Pins for the oracle's bit-level pre-packing (2+4 split, 32-bit words).

The TC-FPx article ("kernel solution redesign") describes the idea: each 6-bit
weight is split into a 2-bit and a 4-bit piece, the pieces are pre-packed
offline into aligned 32-bit words, and the order of fragments is arranged so
that many weights are rebuilt in registers in parallel.  The concrete layout is
this project's own (version 1); what pins it is that the bit-splice rebuild --
word rotations and masks, done here in numpy independently of the oracle's
scatter/gather code -- turns the packed words back into the fp16 pattern
(c & 0x20) << 10 | (c & 0x1F) << 8 of every code.
"""
import numpy as np
import pytest

TILE_BYTES = 6144


def splice_dequant(packed: np.ndarray, N: int, K: int) -> np.ndarray:
    """Rebuild fp16 patterns of decode(c) * 2^-12 from packed words using only
    word rotations and masks: output pair j (columns 2j, 2j+1) of a row is
        rotl(H[j//8], 12 - 2*(j%8)) & 0x90009000  |  shift(L[j//4], 8 - 4*(j%4)) & 0x0F000F00
    where H / L are the row's hi / lo words."""
    words = packed.view("<u4")
    out = np.zeros((N, K), dtype=np.uint16)
    KT = K // 64
    for nt in range(N // 128):
        for kt in range(KT):
            base = (nt * KT + kt) * TILE_BYTES // 4
            r = np.arange(128)
            L = np.stack([words[base + (q // 4) * 512 + r * 4 + (q % 4)] for q in range(8)], axis=1)
            H = np.stack([words[base + 1024 + r * 4 + p] for p in range(4)], axis=1)
            L = L.astype(np.uint64)
            H = H.astype(np.uint64)
            for j in range(32):
                h = H[:, j // 8]
                rot = (12 - 2 * (j % 8)) % 32
                hr = ((h << np.uint64(rot)) | (h >> np.uint64(32 - rot))) & np.uint64(0xFFFFFFFF) if rot else h
                sh = 8 - 4 * (j % 4)
                lw = L[:, j // 4]
                lr = ((lw << np.uint64(sh)) if sh >= 0 else (lw >> np.uint64(-sh))) & np.uint64(0xFFFFFFFF)
                w = (hr & np.uint64(0x90009000)) | (lr & np.uint64(0x0F000F00))
                out[nt * 128:(nt + 1) * 128, kt * 64 + 2 * j] = (w & np.uint64(0xFFFF)).astype(np.uint16)
                out[nt * 128:(nt + 1) * 128, kt * 64 + 2 * j + 1] = (w >> np.uint64(16)).astype(np.uint16)
    return out


def closed_form_pattern(codes: np.ndarray) -> np.ndarray:
    c = codes.astype(np.uint16)
    return ((c & 0x20) << 10) | ((c & 0x1F) << 8)


@pytest.mark.parametrize("N,K,seed", [(128, 64, 0), (256, 512, 1), (384, 192, 2)])
def test_splice_of_packed_gives_closed_form(orc, N, K, seed):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 64, size=(N, K), dtype=np.uint8)
    packed = orc.prepack(codes)
    assert packed.size == N * K * 3 // 4
    assert np.array_equal(splice_dequant(packed, N, K), closed_form_pattern(codes))


def test_all_64_codes_every_position(orc):
    N, K = 128, 128
    codes = ((np.arange(N)[:, None] * 7 + np.arange(K)[None, :]) % 64).astype(np.uint8)
    packed = orc.prepack(codes)
    assert np.array_equal(splice_dequant(packed, N, K), closed_form_pattern(codes))
    assert np.array_equal(orc.unpack(packed, N, K), codes)


def test_one_hot_probe(orc):
    """A single all-ones code at (n, k) sets exactly six bits, all inside tile
    (n//128, k//64) and inside the 48 bytes owned by row n%128 (two 16-byte
    lo units at (u*2048 + r*16), one 16-byte hi unit at 4096 + r*16)."""
    N, K = 256, 128
    KT = K // 64
    rng = np.random.default_rng(5)
    probes = [(0, 0), (127, 63), (128, 64), (255, 127), (5, 70)] + \
             [(int(a), int(b)) for a, b in zip(rng.integers(0, N, 40), rng.integers(0, K, 40))]
    for n, k in probes:
        codes = np.zeros((N, K), dtype=np.uint8)
        codes[n, k] = 0x3F
        packed = orc.prepack(codes)
        bits = np.unpackbits(packed, bitorder="little")
        where = np.nonzero(bits)[0]
        assert where.size == 6
        tile = (n // 128) * KT + k // 64
        byte = where // 8 - tile * TILE_BYTES
        assert (byte >= 0).all() and (byte < TILE_BYTES).all()
        r = n % 128
        owned = set(range(r * 16, r * 16 + 16)) | set(range(2048 + r * 16, 2048 + r * 16 + 16)) | \
            set(range(4096 + r * 16, 4096 + r * 16 + 16))
        assert set(byte.tolist()) <= owned
        # four lo bits in the lo units, two hi bits in the hi unit
        assert sum(1 for b in byte if b >= 4096) == 2


def test_round_trip_random(orc):
    rng = np.random.default_rng(9)
    codes = rng.integers(0, 64, size=(256, 640), dtype=np.uint8)
    assert np.array_equal(orc.unpack(orc.prepack(codes), 256, 640), codes)


def test_prepack_rejects_ragged(orc):
    with pytest.raises(orc.OracleError):
        orc.prepack(np.zeros((100, 64), dtype=np.uint8))
    with pytest.raises(orc.OracleError):
        orc.prepack(np.zeros((128, 96), dtype=np.uint8))


def test_dequant_closed_form(orc):
    rng = np.random.default_rng(2)
    N, K = 128, 128
    codes = rng.integers(0, 64, size=(N, K), dtype=np.uint8)
    scales = (2.0 ** rng.uniform(-10, 2, N)).astype(np.float16)
    packed = orc.prepack(codes)
    from tests.test_oracle_decode import closed_form
    vals = np.array([float(closed_form(c)) for c in range(64)])
    vals[0x20] = -0.0
    ref_plain = vals[codes].astype(np.float16).view(np.uint16)
    assert np.array_equal(orc.dequant(packed, None, N, K), ref_plain)
    ref_scaled = (vals[codes] * scales.astype(np.float64)[:, None]).astype(np.float16).view(np.uint16)
    assert np.array_equal(orc.dequant(packed, scales.view(np.uint16), N, K), ref_scaled)
