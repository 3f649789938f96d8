"""The C-ABI library loads and exports every entry point include/fp6.h declares;
argument validation happens on the host before any CUDA call (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from weight_only_quantized_fp6_b200 import _lib, build
    build.build_library()
    return _lib.load()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "fp6.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b((?:fp[6x]|s24)_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n


def test_binding_covers_header():
    from weight_only_quantized_fp6_b200 import _lib
    assert set(declared_functions()) == set(_lib.SIGNATURES)


def declared_arities():
    """Number of parameters of every function include/fp6.h declares."""
    src = open(os.path.join(ROOT, "include", "fp6.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = {}
    for m in re.finditer(r"\b((?:fp[6x]|s24)_[a-z_0-9]+)\s*\(([^)]*)\)\s*;", src):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else len(params.split(","))
    return out


def test_binding_argument_counts_match_header():
    """The ctypes table passes exactly as many arguments as each C
    declaration takes."""
    from weight_only_quantized_fp6_b200 import _lib
    ar = declared_arities()
    assert set(ar) == set(_lib.SIGNATURES)
    for name, (_, args) in _lib.SIGNATURES.items():
        assert len(args) == ar[name], (name, len(args), ar[name])


def test_status_strings(lib):
    from weight_only_quantized_fp6_b200 import _lib
    for code, name in _lib.STATUS.items():
        assert lib.fp6_status_string(code).decode() == name


def test_packed_bytes(lib):
    assert lib.fp6_packed_bytes(8192, 8192) == 50331648
    assert lib.fp6_packed_bytes(256, 512) == 98304
    assert lib.fp6_packed_bytes(100, 64) == 0
    assert lib.fp6_packed_bytes(128, 96) == 0
    assert lib.fp6_packed_bytes(0, 64) == 0


def test_host_side_validation(lib):
    P = ctypes.c_void_p
    ok_ptr = P(1 << 20)        # 16-byte aligned fake addresses: never dereferenced,
    bad_ptr = P((1 << 20) + 2)  # validation fails before any launch
    # unsupported shapes
    assert lib.fp6_linear(ok_ptr, ok_ptr, ok_ptr, 4, 100, 64, ok_ptr, None, 0, None) == 2
    assert lib.fp6_linear(ok_ptr, ok_ptr, ok_ptr, 4, 128, 96, ok_ptr, None, 0, None) == 2
    assert lib.fp6_prepack(ok_ptr, 128, 100, ok_ptr, 1 << 20, None) == 2
    assert lib.fp6_dequant(ok_ptr, None, 130, 64, ok_ptr, None) == 2
    # negative sizes
    assert lib.fp6_linear(ok_ptr, ok_ptr, ok_ptr, -1, 128, 64, ok_ptr, None, 0, None) == 1
    assert lib.fp6_quantize(ok_ptr, -3, 64, ok_ptr, ok_ptr, None) == 1
    # misaligned pointers
    assert lib.fp6_linear(bad_ptr, ok_ptr, ok_ptr, 4, 128, 64, ok_ptr, None, 0, None) == 3
    assert lib.fp6_linear(ok_ptr, ok_ptr, ok_ptr, 4, 128, 64, bad_ptr, None, 0, None) == 3
    assert lib.fp6_prepack(bad_ptr, 128, 64, ok_ptr, 6144, None) == 3
    assert lib.fp6_dequant(ok_ptr, bad_ptr, 128, 64, ok_ptr, None) == 3
    # null pointers and short buffers
    assert lib.fp6_linear(None, ok_ptr, ok_ptr, 4, 128, 64, ok_ptr, None, 0, None) == 1
    assert lib.fp6_prepack(ok_ptr, 128, 64, ok_ptr, 6143, None) == 1
    # empty problems are no-ops
    assert lib.fp6_linear(None, None, None, 0, 128, 64, ok_ptr, None, 0, None) == 0
    assert lib.fp6_prepack(None, 0, 64, None, 0, None) == 0
    assert lib.fp6_quantize(None, 0, 64, None, None, None) == 0


def test_fpx_packed_bytes_and_validation(lib):
    P = ctypes.c_void_p
    ok_ptr = P(1 << 20)
    assert lib.fpx_packed_bytes(0, 8192, 8192) == 50331648      # e3m2
    assert lib.fpx_packed_bytes(1, 8192, 8192) == 50331648      # e2m3
    assert lib.fpx_packed_bytes(2, 8192, 8192) == 33554432      # e2m1: half a byte per weight
    assert lib.fpx_packed_bytes(3, 8192, 8192) == 41943040      # e2m2: five eighths of a byte
    assert lib.fpx_packed_bytes(2, 128, 96) == 0
    assert lib.fpx_packed_bytes(4, 128, 64) == 0                # unknown format
    assert lib.fpx_packed_bytes(-1, 128, 64) == 0
    # unknown format: an argument error before anything else
    assert lib.fpx_linear(4, ok_ptr, ok_ptr, ok_ptr, 4, 128, 64, ok_ptr, None, 0, None) == 1
    assert lib.fpx_quantize(7, ok_ptr, 128, 64, ok_ptr, ok_ptr, None) == 1
    assert lib.fpx_prepack(-1, ok_ptr, 128, 64, ok_ptr, 1 << 20, None) == 1
    assert lib.fpx_dequant(4, ok_ptr, None, 128, 64, ok_ptr, None) == 1
    # the shape and buffer rules of the fp6 entry points, per format
    for fmt in (0, 1, 2, 3):
        assert lib.fpx_linear(fmt, ok_ptr, ok_ptr, ok_ptr, 4, 100, 64, ok_ptr, None, 0, None) == 2
        assert lib.fpx_prepack(fmt, ok_ptr, 128, 100, ok_ptr, 1 << 20, None) == 2
        assert lib.fpx_linear(fmt, ok_ptr, ok_ptr, ok_ptr, 4, 128, 64, P((1 << 20) + 8), None, 0, None) == 3
        assert lib.fpx_linear(fmt, None, None, None, 0, 128, 64, ok_ptr, None, 0, None) == 0
    assert lib.fpx_prepack(2, ok_ptr, 128, 64, ok_ptr, 4095, None) == 1   # short buffer (needs 4096)
    assert lib.fpx_prepack(1, ok_ptr, 128, 64, ok_ptr, 6143, None) == 1
    assert lib.fpx_prepack(3, ok_ptr, 128, 64, ok_ptr, 5119, None) == 1


def test_python_rejects_unknown_format():
    import weight_only_quantized_fp6_b200 as fp6
    with pytest.raises(ValueError):
        fp6.packed_bytes(128, 64, fmt=5)


def test_oracle_is_not_linked_into_the_library():
    """The product library never references the oracle."""
    from weight_only_quantized_fp6_b200 import build
    for f in build.SOURCES + build.HEADERS:
        text = open(f).read()
        assert "oracle" not in text.lower(), f
    pkg = os.path.join(ROOT, "weight_only_quantized_fp6_b200")
    for name in os.listdir(pkg):
        if name.endswith(".py"):
            assert "import oracle" not in open(os.path.join(pkg, name)).read(), name


def plan(lib, M, N, K, sms=148):
    out = (ctypes.c_int64 * 7)()
    assert lib.fp6_linear_plan_for_sms(M, N, K, sms, out) == 0
    return {"ncol": out[0], "stages": out[1], "grid": out[2], "tiles": out[3], "total": out[4], "T": out[5],
            "wave": out[6]}


def test_plan_token_tiles_and_steps(lib):
    """Token-tile width by M (16, 32, 64 for the decode kernel; 128, 256
    beyond), the widest step that divides K / 64, and a grid of at most one
    CTA per SM and per step."""
    for M, ncol in [(1, 16), (16, 16), (17, 32), (32, 32), (33, 64), (64, 64), (65, 128), (128, 128),
                    (129, 256), (4096, 256)]:
        assert plan(lib, M, 8192, 8192)["ncol"] == ncol, M
    assert plan(lib, 1, 8192, 8192)["T"] == 2
    assert plan(lib, 1, 8192, 64 * 3)["T"] == 1            # three column tiles: odd, one tile per step
    p = plan(lib, 1, 128, 64)
    assert p["total"] == 1 and p["grid"] == 1               # never more CTAs than steps
    p = plan(lib, 1, 8192, 8192)
    assert p["grid"] == 148 and p["tiles"] == 64 and p["total"] == 64 * 64
    assert plan(lib, 16, 8192, 8192, sms=132)["grid"] == 132


def test_plan_wave_schedule_rule(lib):
    """Whole tiles per CTA only with at least as many tiles as SMs and a last
    wave at least 95 % full; every CTA then has a tile."""
    cases = [
        (4096, 28672, 8192, 1),    # 3584 tiles: 25 waves, 3.3 % idle
        (4096, 8192, 28672, 1),    # 1024 tiles: 7 waves, 1.4 % idle
        (4096, 21504, 7168, 1),    # 2688 tiles: 19 waves, 4.6 % idle
        (1024, 28672, 8192, 0),    # 896 tiles: 7 waves, 13.5 % idle
        (1024, 8192, 28672, 0),    # 256 tiles: 2 waves
        (256, 28672, 8192, 0),     # 224 tiles
        (300, 18944, 128, 1),      # 296 tiles: 2 waves, exactly full
        (16, 57344, 8192, 0),      # decode kernel: never
    ]
    for M, N, K, wave in cases:
        p = plan(lib, M, N, K)
        assert p["wave"] == wave, (M, N, K)
        if wave:
            assert p["grid"] == 148 and p["tiles"] >= 148
            waves = -(-p["tiles"] // 148)
            assert waves * 148 * 100 <= p["tiles"] * 105


def test_plan_for_sms_rejects_bad_arguments(lib):
    out = (ctypes.c_int64 * 7)()
    assert lib.fp6_linear_plan_for_sms(1, 8192, 8192, 0, out) == 1
    assert lib.fp6_linear_plan_for_sms(-1, 8192, 8192, 148, out) == 1
    assert lib.fp6_linear_plan_for_sms(1, 100, 8192, 148, out) == 2
    assert lib.fp6_linear_plan_for_sms(1, 8192, 8192, 148, None) == 1
    # more pipeline steps than the kernels count (2^23 row tiles x 2^26 token
    # tiles x 2^23 steps would overflow 64-bit step arithmetic): rejected on the
    # host, before any arithmetic on them
    assert lib.fp6_linear_plan_for_sms(2 ** 31 - 1, 2 ** 30, 2 ** 30, 148, out) == 2
    assert lib.fp6_linear_workspace_bytes(2 ** 31 - 1, 2 ** 30, 2 ** 30) == 0
