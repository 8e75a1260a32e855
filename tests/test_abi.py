"""The C-ABI library: it loads, exports every symbol include/mx.h declares, and rejects bad
arguments on the host before any CUDA call (so these run without a GPU)."""
import ctypes
import os
import re

import numpy as np
import pytest

from mxfp8_block_scaled_07_b200 import build as mxbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mx.h")


@pytest.fixture(scope="module")
def L():
    mxbuild.build()
    from mxfp8_block_scaled_07_b200 import mx

    return mx.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mx_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("mx_quantize", "mx_swizzle_scales", "mx_gemm", "mx_grouped_gemm", "mx_grid_equal",
                     "mx_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings(L):
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert L.mx_status_string(code)
    assert L.mx_status_string(0) == b"MX_OK"


def test_swizzled_scale_bytes(L):
    assert L.mx_swizzled_scale_bytes(0, 0) == 0
    assert L.mx_swizzled_scale_bytes(1, 1) == 512
    assert L.mx_swizzled_scale_bytes(128, 4) == 512
    assert L.mx_swizzled_scale_bytes(129, 5) == 256 * 8
    assert L.mx_swizzled_scale_bytes(24576, 128) == 24576 * 128
    assert L.mx_swizzled_scale_bytes(-1, 4) == -1


FAKE = ctypes.c_void_p(0x10000)       # never dereferenced: every call below fails validation first
FAKE_ODD = ctypes.c_void_p(0x10008)


def test_grouped_scale_bytes_match_per_group_layouts(L):
    """The binding's grouped size (padded rows summed once) equals the sum of the library's size
    of every group's own layout."""
    from mxfp8_block_scaled_07_b200 import mx

    g = np.random.default_rng(3)
    for _ in range(100):
        groups = [int(r) for r in g.choice([0, 1, 127, 128, 129, 255, 256, 300, 1000], g.integers(1, 20))]
        kb = int(g.choice([1, 3, 4, 13, 24, 64, 130]))
        assert mx.grouped_swizzled_scale_bytes(groups, kb) == sum(L.mx_swizzled_scale_bytes(r, kb) for r in groups)


def test_quantize_argument_errors(L):
    q = L.mx_quantize
    assert q(FAKE, 64, 64, 64, 0, FAKE, FAKE, FAKE, FAKE, None) == -1           # no direction
    assert q(FAKE, 64, 64, 64, 8, FAKE, FAKE, FAKE, FAKE, None) == -1           # unknown flag
    assert q(None, 64, 64, 64, 1, FAKE, FAKE, None, None, None) == -1           # null input
    assert q(FAKE, 64, 64, 64, 1, None, FAKE, None, None, None) == -1           # null output
    assert q(FAKE, 64, 64, 64, 2, None, None, FAKE, None, None) == -1
    assert q(FAKE, -1, 64, 64, 1, FAKE, FAKE, None, None, None) == -1
    assert q(FAKE, 64, 48, 64, 1, FAKE, FAKE, None, None, None) == -2           # K % 32
    assert q(FAKE, 48, 64, 64, 2, None, None, FAKE, FAKE, None) == -2           # M % 32 for colwise
    assert q(FAKE, 64, 64, 32, 1, FAKE, FAKE, None, None, None) == -2           # ld_x < K
    assert q(FAKE_ODD, 64, 64, 64, 1, FAKE, FAKE, None, None, None) == -3       # misaligned x
    assert q(FAKE, 64, 64, 68, 1, FAKE, FAKE, None, None, None) == -3           # ld_x % 8
    assert q(FAKE, 64, 64, 64, 1, FAKE_ODD, FAKE, None, None, None) == -3


def test_gemm_argument_errors(L):
    g = L.mx_gemm
    assert g(None, FAKE, FAKE, FAKE, 8, 8, 32, FAKE, 8, 0, None) == -1
    assert g(FAKE, FAKE, FAKE, FAKE, 8, 8, 0, FAKE, 8, 0, None) == -1
    assert g(FAKE, FAKE, FAKE, FAKE, 8, 8, 32, FAKE, 8, 7, None) == -1           # bad dtype
    assert g(FAKE, FAKE, FAKE, FAKE, 8, 8, 48, FAKE, 8, 0, None) == -2           # K % 32
    assert g(FAKE, FAKE, FAKE, FAKE, 8, 16, 32, FAKE, 8, 0, None) == -2          # ld_c < N
    assert g(FAKE, FAKE, FAKE, FAKE, 8, 8, 32, ctypes.c_void_p(0x10002), 8, 0, None) == -3   # f32 misaligned
    assert g(FAKE_ODD, FAKE, FAKE, FAKE, 8, 8, 32, FAKE, 8, 0, None) == -3      # operand not 16-byte aligned
    assert g(FAKE, FAKE, FAKE, FAKE, 0, 8, 32, None, 8, 0, None) == 0           # empty: no-op, null allowed
    gg = L.mx_grouped_gemm
    assert gg(FAKE, FAKE, FAKE, FAKE, None, 4, 64, 8, 32, FAKE, 8, 0, None) == -1
    assert gg(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 64, 8, 32, FAKE, 8, 0, None) == -1
    assert gg(FAKE, FAKE, FAKE, FAKE, FAKE, 1025, 64, 8, 32, FAKE, 8, 0, None) == -2
    sq = L.mx_grouped_gemm_swiglu_quant     # (qa, sa, qb, sb, off, G, rows, n_inter, K, h_q, h_s, stream)
    assert sq(FAKE, FAKE, FAKE, FAKE, None, 4, 64, 128, 32, FAKE, FAKE, None) == -1
    assert sq(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 64, 128, 32, FAKE, FAKE, None) == -1
    assert sq(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 64, 96, 32, FAKE, FAKE, None) == -2      # n_inter % 128
    assert sq(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 64, 128, 48, FAKE, FAKE, None) == -2     # K % 32
    assert sq(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 64, 128, 32, FAKE_ODD, FAKE, None) == -3  # h_q alignment
    assert sq(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 64, 128, 32, FAKE, None, None) == -1     # no h_s
    assert sq(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 0, 128, 32, None, None, None) == 0       # empty: no-op
    bq = L.mx_quantize_block128              # (x, M, K, ld_x, pow2, q, scales, stream)
    assert bq(FAKE, -1, 64, 64, 0, FAKE, FAKE, None) == -1
    assert bq(FAKE, 64, 48, 64, 0, FAKE, FAKE, None) == -2                      # K % 32
    assert bq(FAKE, 64, 64, 32, 0, FAKE, FAKE, None) == -2                      # ld_x < K
    assert bq(FAKE_ODD, 64, 64, 64, 0, FAKE, FAKE, None) == -3                  # x alignment
    assert bq(FAKE, 64, 64, 64, 1, FAKE, ctypes.c_void_p(0x10002), None) == -3  # scales alignment
    assert bq(None, 64, 64, 64, 0, FAKE, FAKE, None) == -1
    assert bq(None, 0, 64, 64, 0, None, None, None) == 0                        # empty: no-op


def test_swizzle_and_grid_equal_argument_errors(L):
    s = L.mx_swizzle_scales
    assert s(None, 4, 4, None, 0, FAKE, None) == -1
    assert s(FAKE, 4, 4, None, 0, FAKE_ODD, None) == -3
    rows = (ctypes.c_int64 * 2)(3, 4)
    assert s(FAKE, 8, 4, ctypes.cast(rows, ctypes.c_void_p), 2, FAKE, None) == -2   # groups do not sum to rows
    neg = (ctypes.c_int64 * 2)(-1, 8)
    assert s(FAKE, 7, 4, ctypes.cast(neg, ctypes.c_void_p), 2, FAKE, None) == -1
    assert s(None, 0, 4, None, 0, None, None) == 0        # empty: a no-op, NULL pointers allowed
    assert s(None, 4, 0, None, 0, None, None) == 0
    e = L.mx_grid_equal
    assert e(FAKE, FAKE, 16, None, FAKE, None) == -1
    assert e(FAKE, FAKE, -1, FAKE, FAKE, None) == -1
    assert e(None, FAKE, 16, FAKE, FAKE, None) == -1
    assert L.mx_device_error(None) == -1


def test_multi_calls_validate_every_entry(L):
    from mxfp8_block_scaled_07_b200 import mx

    assert L.mx_quantize_multi(None, 3, 1, None) == -1
    assert L.mx_quantize_multi(None, 0, 1, None) == 0
    arr = (mx.QuantTensor * 2)(mx.QuantTensor(0x10000, 64, 64, 64, 0x10000, 0x10000, None, None),
                               mx.QuantTensor(0x10000, 64, 48, 64, 0x10000, 0x10000, None, None))
    assert L.mx_quantize_multi(ctypes.cast(arr, ctypes.c_void_p), 2, 1, None) == -2      # 2nd: K % 32
    arr[1] = mx.QuantTensor(0x10008, 64, 64, 64, 0x10000, 0x10000, None, None)
    assert L.mx_quantize_multi(ctypes.cast(arr, ctypes.c_void_p), 2, 1, None) == -3      # 2nd: misaligned
    assert L.mx_quantize_multi(ctypes.cast(arr, ctypes.c_void_p), 2, 0, None) == -1      # no direction
    pairs = (mx.ComparePair * 2)(mx.ComparePair(0x10000, 0x10000, 16), mx.ComparePair(None, 0x10000, 4))
    assert L.mx_grid_equal_multi(ctypes.cast(pairs, ctypes.c_void_p), 2, FAKE, FAKE, None) == -1
    assert L.mx_grid_equal_multi(ctypes.cast(pairs, ctypes.c_void_p), 1, None, FAKE, None) == -1
    assert L.mx_grid_equal_multi(None, 0, None, None, None) == 0


def test_quantize_compare_multi_validates_before_launching(L):
    from mxfp8_block_scaled_07_b200 import mx

    P = ctypes.c_void_p
    good = mx.QuantTensor(0x10000, 64, 64, 64, 0x10000, 0x10000, None, None)
    arr = (mx.QuantTensor * 2)(good, good)
    refs = (mx.GridRef * 2)(mx.GridRef(0x10000, 0x10000), mx.GridRef(0x10000, 0x10000))
    A, R = ctypes.cast(arr, P), ctypes.cast(refs, P)
    assert L.mx_quantize_compare_multi(None, None, 0, None, None, None) == 0
    assert L.mx_quantize_compare_multi(A, R, -1, FAKE, FAKE, None) == -1
    assert L.mx_quantize_compare_multi(A, None, 2, FAKE, FAKE, None) == -1            # no references
    assert L.mx_quantize_compare_multi(A, R, 2, None, FAKE, None) == -1               # no result array
    refs[1] = mx.GridRef(0x10000, None)
    assert L.mx_quantize_compare_multi(A, R, 2, FAKE, FAKE, None) == -1               # 2nd: no reference scales
    refs[1] = mx.GridRef(0x10008, 0x10000)
    assert L.mx_quantize_compare_multi(A, R, 2, FAKE, FAKE, None) == -3               # 2nd: misaligned reference
    refs[1] = mx.GridRef(0x10000, 0x10000)
    arr[1] = mx.QuantTensor(0x10000, 64, 48, 64, 0x10000, 0x10000, None, None)
    assert L.mx_quantize_compare_multi(A, R, 2, FAKE, FAKE, None) == -2               # 2nd: K % 32
    arr[1] = mx.QuantTensor(0x10000, 0, 64, 64, None, None, None, None)
    refs[1] = mx.GridRef(None, None)                                                   # empty: refs unused
    assert L.mx_quantize_compare_multi(A, R, 1, FAKE, FAKE, None) != -1


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    from mxfp8_block_scaled_07_b200 import mx

    monkeypatch.setattr(mx, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(mx, "_lib", None)
    with pytest.raises(ImportError):
        mx.lib()
