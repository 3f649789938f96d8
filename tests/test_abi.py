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
    return sorted(set(re.findall(r"\b(fp[6x]_[a-z_0-9]+)\s*\(", src)))


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
    for m in re.finditer(r"\b(fp[6x]_[a-z_0-9]+)\s*\(([^)]*)\)\s*;", src):
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
