"""CPU oracle for the MXFP8 learner/sampler grid -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg (and its
``--impl reference`` arm) may import this package. The product library never does, and the
two share no code: this is a ctypes wrapper around ``mx_oracle.c``, a plain fp64 C
restatement of the MXFP8 rule (OCP MX v1.0: E4M3 elements, one E8M0 power-of-two scale per
32 elements) that the paper "End-to-End MXFP8 Reinforcement Learning on Blackwell"
(arXiv 2610.34915) relies on (Figure 1; Table 1; Table 10, F3 and F6; Table 11).

All arrays are numpy; BF16 tensors are passed as their uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mx_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libmx_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, no fast-math so fp64 stays IEEE)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "mx_oracle.h"))
    ):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_decode.restype = ctypes.c_double
    lib.oracle_e4m3_encode.argtypes = [ctypes.c_double]
    lib.oracle_e4m3_encode.restype = ctypes.c_uint8
    lib.oracle_e4m3_encode_array.argtypes = [P, I64, P]
    lib.oracle_e4m3_encode_array.restype = None
    lib.oracle_e8m0_scale.argtypes = [ctypes.c_double]
    lib.oracle_e8m0_scale.restype = ctypes.c_uint8
    lib.oracle_quantize_rowwise.argtypes = [P, I64, I64, I64, P, P]
    lib.oracle_quantize_rowwise.restype = ctypes.c_int
    lib.oracle_quantize_colwise.argtypes = [P, I64, I64, I64, P, P]
    lib.oracle_quantize_colwise.restype = ctypes.c_int
    lib.oracle_dequantize.argtypes = [P, P, I64, I64, P]
    lib.oracle_dequantize.restype = None
    lib.oracle_swizzled_size.argtypes = [I64, I64, P, I64]
    lib.oracle_swizzled_size.restype = I64
    lib.oracle_swizzle.argtypes = [P, I64, I64, P, I64, P]
    lib.oracle_swizzle.restype = None
    lib.oracle_gemm.argtypes = [P, P, P, P, I64, I64, I64, P, P]
    lib.oracle_gemm.restype = None
    lib.oracle_grouped_gemm.argtypes = [P, P, P, P, P, I64, I64, I64, P, P]
    lib.oracle_grouped_gemm.restype = None
    lib.oracle_quantize_block128.argtypes = [P, I64, I64, I64, ctypes.c_int, P, P]
    lib.oracle_quantize_block128.restype = None
    lib.oracle_swiglu_quantize.argtypes = [P, I64, I64, P, P, P]
    lib.oracle_swiglu_quantize.restype = ctypes.c_int
    lib.oracle_grid_equal.argtypes = [P, P, I64, P, P]
    lib.oracle_grid_equal.restype = None
    _lib = lib
    return lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _bits(x) -> np.ndarray:
    """BF16 input as a C-contiguous uint16 array of bit patterns (accepts torch or numpy)."""
    try:
        import torch

        if isinstance(x, torch.Tensor):
            assert x.dtype == torch.bfloat16
            return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))
    except ImportError:  # pragma: no cover
        pass
    x = np.asarray(x)
    assert x.dtype == np.uint16
    return np.ascontiguousarray(x)


def e4m3_decode(code: int) -> float:
    return _load().oracle_e4m3_decode(int(code))


def e4m3_encode(v: float) -> int:
    return int(_load().oracle_e4m3_encode(float(v)))


def e4m3_encode_array(v) -> np.ndarray:
    v = np.ascontiguousarray(v, np.float64).reshape(-1)
    out = np.empty(v.size, np.uint8)
    _load().oracle_e4m3_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def e8m0_scale(amax: float) -> int:
    return int(_load().oracle_e8m0_scale(float(amax)))


def quantize_rowwise(x):
    """x: BF16 [M, K] -> (q uint8 [M, K], s uint8 [M, K/32])."""
    xb = _bits(x)
    M, K = xb.shape
    q = np.empty((M, K), np.uint8)
    s = np.empty((M, K // 32), np.uint8)
    rc = _load().oracle_quantize_rowwise(_ptr(xb), M, K, K, _ptr(q), _ptr(s))
    if rc != 0:
        raise ValueError("K must be a multiple of 32")
    return q, s


def quantize_colwise(x):
    """x: BF16 [M, K] -> (qT uint8 [K, M], sT uint8 [K, M/32])."""
    xb = _bits(x)
    M, K = xb.shape
    qT = np.empty((K, M), np.uint8)
    sT = np.empty((K, M // 32), np.uint8)
    rc = _load().oracle_quantize_colwise(_ptr(xb), M, K, K, _ptr(qT), _ptr(sT))
    if rc != 0:
        raise ValueError("M must be a multiple of 32")
    return qT, sT


def dequantize(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, np.uint8)
    s = np.ascontiguousarray(s, np.uint8)
    rows, K = q.shape
    out = np.empty((rows, K), np.float64)
    _load().oracle_dequantize(_ptr(q), _ptr(s), rows, K, _ptr(out))
    return out


def swizzled_size(rows: int, cols: int, group_rows=None) -> int:
    if group_rows is None:
        return int(_load().oracle_swizzled_size(rows, cols, None, 0))
    g = np.ascontiguousarray(group_rows, np.int64)
    return int(_load().oracle_swizzled_size(rows, cols, _ptr(g), len(g)))


def swizzle(s: np.ndarray, group_rows=None) -> np.ndarray:
    s = np.ascontiguousarray(s, np.uint8)
    rows, cols = s.shape
    out = np.empty(swizzled_size(rows, cols, group_rows), np.uint8)
    if group_rows is None:
        _load().oracle_swizzle(_ptr(s), rows, cols, None, 0, _ptr(out))
    else:
        g = np.ascontiguousarray(group_rows, np.int64)
        assert int(g.sum()) == rows
        _load().oracle_swizzle(_ptr(s), rows, cols, _ptr(g), len(g), _ptr(out))
    return out


def gemm(qa, sa, qb, sb):
    """C = dq(A) . dq(B)^T in fp64 with raw scales; returns (C, sum_k |a_k b_k|)."""
    qa, sa, qb, sb = (np.ascontiguousarray(t, np.uint8) for t in (qa, sa, qb, sb))
    M, K = qa.shape
    N = qb.shape[0]
    assert qb.shape[1] == K and sa.shape == (M, K // 32) and sb.shape == (N, K // 32)
    c = np.empty((M, N), np.float64)
    a = np.empty((M, N), np.float64)
    _load().oracle_gemm(_ptr(qa), _ptr(sa), _ptr(qb), _ptr(sb), M, N, K, _ptr(c), _ptr(a))
    return c, a


def grouped_gemm(qa, sa, qb, sb, row_offsets):
    """Per-group GEMM: rows [off[g], off[g+1]) of A against qb[g] ([G, N, K])."""
    qa, sa, qb, sb = (np.ascontiguousarray(t, np.uint8) for t in (qa, sa, qb, sb))
    off = np.ascontiguousarray(row_offsets, np.int64)
    G, N, K = qb.shape
    assert len(off) == G + 1 and off[-1] == qa.shape[0]
    c = np.empty((qa.shape[0], N), np.float64)
    a = np.empty((qa.shape[0], N), np.float64)
    _load().oracle_grouped_gemm(_ptr(qa), _ptr(sa), _ptr(qb), _ptr(sb), _ptr(off), G, N, K, _ptr(c), _ptr(a))
    return c, a


def quantize_block128(x, pow2: bool):
    """x: BF16 [M, K] -> (q uint8 [M, K], scales float32 [ceil(M/128), ceil(K/128)]): FP8 blockwise
    with FP32 scales (pow2=False) or power-of-two scales (pow2=True)."""
    xb = _bits(x)
    M, K = xb.shape
    q = np.empty((M, K), np.uint8)
    s = np.empty(((M + 127) // 128, (K + 127) // 128), np.float32)
    _load().oracle_quantize_block128(_ptr(xb), M, K, K, 1 if pow2 else 0, _ptr(q), _ptr(s))
    return q, s


def swiglu_quantize(gu):
    """gu: fp64 [rows, 2n] (gate features, then up features) -> (h fp64 [rows, n], q uint8
    [rows, n], s uint8 [rows, n/32]): h = silu(gate) * up, then the rowwise MXFP8 rule on h."""
    gu = np.ascontiguousarray(gu, np.float64)
    rows, n2 = gu.shape
    n = n2 // 2
    h = np.empty((rows, n), np.float64)
    q = np.empty((rows, n), np.uint8)
    s = np.empty((rows, n // 32), np.uint8)
    if _load().oracle_swiglu_quantize(_ptr(gu), rows, n, _ptr(h), _ptr(q), _ptr(s)) != 0:
        raise ValueError("n must be a multiple of 32")
    return h, q, s


def grid_equal(a: np.ndarray, b: np.ndarray):
    a = np.ascontiguousarray(a, np.uint8).reshape(-1)
    b = np.ascontiguousarray(b, np.uint8).reshape(-1)
    assert a.size == b.size
    cnt = np.zeros(1, np.uint64)
    first = np.zeros(1, np.int64)
    _load().oracle_grid_equal(_ptr(a), _ptr(b), a.size, _ptr(cnt), _ptr(first))
    return int(cnt[0]), int(first[0])
