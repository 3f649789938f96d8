"""Stored packed weights: the 64-byte blob header (include/fp6.h), written and
checked by the library on the host alone, read back here field by field with
an independent reader; mismatched layouts are rejected with
FP6_ERR_LAYOUT_VERSION."""
import ctypes
import struct

import pytest

LAYOUT_ERR = 7
# format: (layout version, bytes per 128 x 64 tile, packed bytes per weight x 8)
FORMATS = {0: (2, 6144, 6), 1: (2, 6144, 6), 2: (1, 4096, 4), 3: (1, 5120, 5), 4: (1, 3072, 3)}


@pytest.fixture(scope="module")
def lib():
    from weight_only_quantized_fp6_b200 import build, _lib
    build.build_library()
    return _lib.load()


def header(lib, fmt, N, K):
    buf = ctypes.create_string_buffer(64)
    st = lib.fp6_packed_header(fmt, N, K, buf)
    return st, buf.raw


@pytest.mark.parametrize("fmt", sorted(FORMATS))
def test_header_fields(lib, fmt):
    N, K = 8192, 28672
    st, h = header(lib, fmt, N, K)
    assert st == 0
    magic, version, f, hbytes, n, k, tr, tc, tb, sb, payload, pad = struct.unpack("<4sIIIqqIIIIQQ", h)
    ver, tile_bytes, eighths = FORMATS[fmt]
    assert (magic, version, f, hbytes) == (b"FP6W", ver, fmt, 64)
    assert (n, k, tr, tc, tb, sb, pad) == (N, K, 128, 64, tile_bytes, 2, 0)
    assert payload == N * K * eighths // 8 == (N // 128) * (K // 64) * tile_bytes
    assert lib.fp6_packed_header_check(h, fmt, N, K) == 0


@pytest.mark.parametrize("fmt", sorted(FORMATS))
def test_mismatches_are_rejected(lib, fmt):
    N, K = 1024, 2048
    _, h = header(lib, fmt, N, K)
    for off, val in [(0, b"FP5W"), (4, struct.pack("<I", FORMATS[fmt][0] + 1)),   # magic, newer layout
                     (4, struct.pack("<I", FORMATS[fmt][0] - 1)),                   # older layout
                     (12, struct.pack("<I", 128)), (40, struct.pack("<I", 6000)),
                     (48, struct.pack("<Q", 7)), (56, b"\x01")]:
        bad = h[:off] + val + h[off + len(val):]
        assert lib.fp6_packed_header_check(bad, fmt, N, K) == LAYOUT_ERR, off
    assert lib.fp6_packed_header_check(h, fmt, N + 128, K) == LAYOUT_ERR       # another shape
    assert lib.fp6_packed_header_check(h, fmt, N, K + 64) == LAYOUT_ERR
    other = (fmt + 2) % 5
    if FORMATS[other] != FORMATS[fmt] or other in (2, 3, 4):
        assert lib.fp6_packed_header_check(h, other, N, K) == LAYOUT_ERR        # another format
    assert lib.fp6_packed_header_check(h, fmt, 100, K) == LAYOUT_ERR             # a shape no blob has


def test_argument_errors(lib):
    buf = ctypes.create_string_buffer(64)
    assert lib.fp6_packed_header(5, 128, 64, buf) == 1
    assert lib.fp6_packed_header(0, 128, 64, None) == 1
    assert lib.fp6_packed_header(0, 100, 64, buf) == 2
    assert lib.fp6_packed_header_check(None, 0, 128, 64) == 1
    assert lib.fp6_packed_header_check(buf, 9, 128, 64) == 1


def test_e2m3_and_e3m2_share_the_layout_but_not_the_header(lib):
    _, h0 = header(lib, 0, 256, 256)
    _, h1 = header(lib, 1, 256, 256)
    assert h0[4:8] == h1[4:8] and h0[8:12] != h1[8:12]
    assert lib.fp6_packed_header_check(h0, 1, 256, 256) == LAYOUT_ERR
