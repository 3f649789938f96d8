"""Pins for the oracle's bit-level pre-packing (32-bit fragment words).

The TC-FPx article ("kernel solution redesign") describes the idea: each 6-bit
weight is cut into pieces that are pre-packed offline into aligned 32-bit
words, in an order that lets registers rebuild many weights in parallel.  The
concrete cut and order are this project's own (layout version 2): of every 16
codes of a row, 12 sit whole in the low six bits of a byte and 4 are cut into
2-bit pieces held in the top two bits of those bytes.  What pins the oracle's
scatter/gather code is an independent reader, written here in numpy the way
the GPU reads the words (whole-word loads, low six bits of each byte, top-bit
gather with shifts and masks), which must recover every code.
"""
import numpy as np
import pytest

TILE_BYTES = 6144


def read_codes(packed: np.ndarray, N: int, K: int) -> np.ndarray:
    """Recover the codes from packed words with word-level operations only:
    for group g of a row (words F[3g], F[3g+1], F[3g+2]), column 16g + 4j + b
    (j < 3) is byte b of F[3g+j] masked to six bits, and column 16g + 12 + b is
    assembled from the top two bits of byte b of the three words."""
    words = packed.view("<u4").astype(np.uint64)
    out = np.zeros((N, K), dtype=np.uint8)
    KT = K // 64
    r = np.arange(128)
    for nt in range(N // 128):
        for kt in range(KT):
            base = (nt * KT + kt) * TILE_BYTES // 4
            F = np.stack([words[base + (w // 4) * 512 + r * 4 + (w % 4)] for w in range(12)], axis=1)
            rows = slice(nt * 128, (nt + 1) * 128)
            for g in range(4):
                f = [F[:, 3 * g + j] for j in range(3)]
                for j in range(3):
                    for b in range(4):
                        out[rows, kt * 64 + 16 * g + 4 * j + b] = (f[j] >> np.uint64(8 * b)) & np.uint64(0x3F)
                # top-bit gather: t = ((F2 & 0xC0..) | (F1 >> 2 & 0x30..) | (F0 >> 4 & 0x0C..)) >> 2
                t = (f[2] & np.uint64(0xC0C0C0C0)) | ((f[1] >> np.uint64(2)) & np.uint64(0x30303030)) | \
                    ((f[0] >> np.uint64(4)) & np.uint64(0x0C0C0C0C))
                t >>= np.uint64(2)
                for b in range(4):
                    out[rows, kt * 64 + 16 * g + 12 + b] = (t >> np.uint64(8 * b)) & np.uint64(0x3F)
    return out


def closed_form_pattern(codes: np.ndarray) -> np.ndarray:
    """fp16 bit pattern of decode(c), from the closed form (every value is exact in fp16)."""
    from tests.test_oracle_decode import closed_form
    vals = np.array([float(closed_form(c)) for c in range(64)])
    vals[0x20] = -0.0
    return vals[codes].astype(np.float16).view(np.uint16)


@pytest.mark.parametrize("N,K,seed", [(128, 64, 0), (256, 512, 1), (384, 192, 2)])
def test_reader_of_packed_gives_codes(orc, N, K, seed):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 64, size=(N, K), dtype=np.uint8)
    packed = orc.prepack(codes)
    assert packed.size == N * K * 3 // 4
    got = read_codes(packed, N, K)
    assert np.array_equal(got, codes)
    assert np.array_equal(closed_form_pattern(got), orc.dequant(packed, None, N, K))


def test_all_64_codes_every_position(orc):
    N, K = 128, 128
    codes = ((np.arange(N)[:, None] * 7 + np.arange(K)[None, :]) % 64).astype(np.uint8)
    packed = orc.prepack(codes)
    assert np.array_equal(read_codes(packed, N, K), codes)
    assert np.array_equal(orc.unpack(packed, N, K), codes)


def test_one_hot_probe(orc):
    """A single all-ones code at (n, k) sets exactly six bits, all inside tile
    (n//128, k//64) and inside the 48 bytes owned by row n%128 (16-byte units
    at u*2048 + r*16, u = 0, 1, 2): for a whole code six low bits of one byte,
    for a cut code the top two bits of three bytes."""
    N, K = 256, 128
    KT = K // 64
    rng = np.random.default_rng(5)
    probes = [(0, 0), (127, 63), (128, 64), (255, 127), (5, 70), (3, 12), (9, 47)] + \
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
        owned = set()
        for u in range(3):
            owned |= set(range(u * 2048 + r * 16, u * 2048 + r * 16 + 16))
        assert set(byte.tolist()) <= owned
        in_byte = sorted((where % 8).tolist())
        if (k % 64) % 16 < 12:
            assert len(set(byte.tolist())) == 1 and in_byte == [0, 1, 2, 3, 4, 5]
        else:
            assert len(set(byte.tolist())) == 3 and in_byte == [6, 6, 6, 7, 7, 7]


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
