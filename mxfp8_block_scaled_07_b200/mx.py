"""Thin Python binding of libmx (include/mx.h) over ctypes.

Argument marshalling only: every step runs in the CUDA kernels of ``libmx.so``. PyTorch
supplies device memory (output tensors are allocated with ``torch.empty`` on the input's
device) and the current stream. There is no fallback: if ``libmx.so`` is missing or a call
fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmx.so")

MX_ROWWISE, MX_COLWISE, MX_SWIZZLE = 1, 2, 4
MX_OUT_F32, MX_OUT_BF16 = 0, 1
_STATUS = {0: "MX_OK", -1: "MX_ERR_ARG", -2: "MX_ERR_SHAPE", -3: "MX_ERR_ALIGN", -4: "MX_ERR_CUDA",
           -5: "MX_ERR_UNSUPPORTED", -6: "MX_ERR_DEVICE"}

_lib = None


class QuantTensor(ctypes.Structure):
    """mx_quant_tensor."""
    _fields_ = [("x", ctypes.c_void_p), ("M", ctypes.c_int64), ("K", ctypes.c_int64), ("ld_x", ctypes.c_int64),
                ("q_row", ctypes.c_void_p), ("s_row", ctypes.c_void_p), ("q_col", ctypes.c_void_p),
                ("s_col", ctypes.c_void_p)]


class GridRef(ctypes.Structure):
    """mx_grid_ref."""
    _fields_ = [("q", ctypes.c_void_p), ("s", ctypes.c_void_p)]


class ComparePair(ctypes.Structure):
    """mx_compare_pair."""
    _fields_ = [("a", ctypes.c_void_p), ("b", ctypes.c_void_p), ("nbytes", ctypes.c_int64)]


class MxError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {_STATUS.get(status, status)}")
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded libmx.so with argument types declared (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libmx.so not built ({LIB_PATH}); run python -m mxfp8_block_scaled_07_b200.build")
    L = ctypes.CDLL(LIB_PATH)
    P, I64, I32, U64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint64
    L.mx_swizzled_scale_bytes.argtypes = [I64, I64]
    L.mx_swizzled_scale_bytes.restype = I64
    L.mx_quantize.argtypes = [P, I64, I64, I64, I32, P, P, P, P, P]
    L.mx_quantize.restype = I32
    L.mx_swizzle_scales.argtypes = [P, I64, I64, P, I64, P, P]
    L.mx_swizzle_scales.restype = I32
    L.mx_gemm.argtypes = [P, P, P, P, I64, I64, I64, P, I64, I32, P]
    L.mx_gemm.restype = I32
    L.mx_quantize_block128.argtypes = [P, I64, I64, I64, I32, P, P, P]
    L.mx_quantize_block128.restype = I32
    L.mx_grouped_gemm_swiglu_quant.argtypes = [P, P, P, P, P, I64, I64, I64, I64, P, P, P]
    L.mx_grouped_gemm_swiglu_quant.restype = I32
    L.mx_grouped_gemm.argtypes = [P, P, P, P, P, I64, I64, I64, I64, P, I64, I32, P]
    L.mx_grouped_gemm.restype = I32
    L.mx_grid_equal.argtypes = [P, P, I64, P, P, P]
    L.mx_grid_equal.restype = I32
    L.mx_quantize_multi.argtypes = [P, I64, I32, P]
    L.mx_quantize_multi.restype = I32
    L.mx_grid_equal_multi.argtypes = [P, I64, P, P, P]
    L.mx_grid_equal_multi.restype = I32
    L.mx_quantize_compare_multi.argtypes = [P, P, I64, P, P, P]
    L.mx_quantize_compare_multi.restype = I32
    L.mx_status_string.argtypes = [I32]
    L.mx_status_string.restype = ctypes.c_char_p
    L.mx_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32)]
    L.mx_device_error.restype = I32
    L.mx_set_wait_timeout_ns.argtypes = [U64]
    L.mx_set_wait_timeout_ns.restype = None
    L.mx_set_gemm_variant.argtypes = [I32]
    L.mx_set_gemm_variant.restype = None
    L.mx_set_quantize_variant.argtypes = [I32]
    L.mx_set_quantize_variant.restype = None
    L.mx_diag_expired_wait.argtypes = [P]
    L.mx_diag_expired_wait.restype = I32
    _lib = L
    return L


def _check(status: int, what: str):
    if status != 0:
        raise MxError(status, what)


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def swizzled_scale_bytes(rows: int, kblocks: int) -> int:
    return int(lib().mx_swizzled_scale_bytes(rows, kblocks))


def grouped_swizzled_scale_bytes(group_rows, kblocks: int) -> int:
    """Bytes of the grouped layout: every group padded to 128 rows on its own (no library call per
    group: the padded row count times the padded K-block count)."""
    rows = sum((int(r) + 127) // 128 * 128 for r in group_rows)
    return swizzled_scale_bytes(rows, kblocks) if rows else 0


def quantize(x: torch.Tensor, rowwise: bool = True, colwise: bool = False, swizzle: bool = True, out=None):
    """mx_quantize on a 2-D BF16 CUDA tensor. Returns (q_row, s_row, q_col, s_col); entries of a
    direction not requested are None. ``out`` may supply the four buffers."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    M, K = x.shape
    flags = (MX_ROWWISE if rowwise else 0) | (MX_COLWISE if colwise else 0) | (MX_SWIZZLE if swizzle else 0)
    dev = x.device
    if out is None:
        u8 = dict(dtype=torch.uint8, device=dev)
        q_row = torch.empty((M, K), **u8) if rowwise else None
        s_row = (torch.empty(swizzled_scale_bytes(M, K // 32), **u8) if swizzle
                 else torch.empty((M, K // 32), **u8)) if rowwise else None
        q_col = torch.empty((K, M), **u8) if colwise else None
        s_col = (torch.empty(swizzled_scale_bytes(K, M // 32), **u8) if swizzle
                 else torch.empty((K, M // 32), **u8)) if colwise else None
    else:
        q_row, s_row, q_col, s_col = out
    st = lib().mx_quantize(_p(x), M, K, x.stride(0), flags, _p(q_row), _p(s_row), _p(q_col), _p(s_col),
                           ctypes.c_void_p(_stream(dev)))
    _check(st, "mx_quantize")
    return q_row, s_row, q_col, s_col


def quant_tensor_array(xs, outs):
    """ctypes array of mx_quant_tensor for tensors xs and their (q_row, s_row, q_col, s_col) outputs."""
    arr = (QuantTensor * len(xs))()
    for i, (x, (q_row, s_row, q_col, s_col)) in enumerate(zip(xs, outs)):
        assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
        arr[i] = QuantTensor(x.data_ptr(), x.shape[0], x.shape[1], x.stride(0),
                             *(t.data_ptr() if t is not None else None for t in (q_row, s_row, q_col, s_col)))
    return arr


def quantize_multi(xs, rowwise: bool = True, colwise: bool = False, swizzle: bool = True, outs=None):
    """mx_quantize_multi over a list of 2-D BF16 CUDA tensors (same flags); returns one
    (q_row, s_row, q_col, s_col) tuple per tensor."""
    if outs is None:
        outs = []
        for x in xs:
            M, K = x.shape
            u8 = dict(dtype=torch.uint8, device=x.device)
            outs.append((
                torch.empty((M, K), **u8) if rowwise else None,
                (torch.empty(swizzled_scale_bytes(M, K // 32), **u8) if swizzle else torch.empty((M, K // 32), **u8))
                if rowwise else None,
                torch.empty((K, M), **u8) if colwise else None,
                (torch.empty(swizzled_scale_bytes(K, M // 32), **u8) if swizzle else torch.empty((K, M // 32), **u8))
                if colwise else None))
    flags = (MX_ROWWISE if rowwise else 0) | (MX_COLWISE if colwise else 0) | (MX_SWIZZLE if swizzle else 0)
    arr = quant_tensor_array(xs, outs)
    dev = xs[0].device if xs else torch.device("cuda")
    st = lib().mx_quantize_multi(ctypes.cast(arr, ctypes.c_void_p), len(xs), flags, ctypes.c_void_p(_stream(dev)))
    _check(st, "mx_quantize_multi")
    return outs


def compare_pair_array(pairs):
    arr = (ComparePair * len(pairs))()
    for i, (a, b) in enumerate(pairs):
        n = a.numel() * a.element_size()
        assert a.is_contiguous() and b.is_contiguous() and b.numel() * b.element_size() == n
        arr[i] = ComparePair(a.data_ptr(), b.data_ptr(), n)
    return arr


def quantize_compare_multi(xs, refs, outs=None, results=None):
    """mx_quantize_compare_multi: the rowwise codes and tensor-core scale layout of every BF16
    tensor in xs (written to outs, as quantize_multi(xs, True, False, True) would), compared byte for
    byte with refs[i] = (q, s_swizzled) in the same pass. Returns (outs, mismatches, first_index);
    the last two are int64 device tensors of 2 len(xs) entries: codes then scales per tensor."""
    n = len(xs)
    dev = xs[0].device if xs else torch.device("cuda")
    if outs is None:
        outs = []
        for x in xs:
            M, K = x.shape
            u8 = dict(dtype=torch.uint8, device=x.device)
            outs.append((torch.empty((M, K), **u8), torch.empty(swizzled_scale_bytes(M, K // 32), **u8), None, None))
    if results is None:
        results = torch.empty((2, max(2 * n, 1)), dtype=torch.int64, device=dev)
    arr = quant_tensor_array(xs, outs)
    ref_arr = (GridRef * max(n, 1))()
    for i, (q, s) in enumerate(refs):
        ref_arr[i] = GridRef(q.data_ptr(), s.data_ptr())
    st = lib().mx_quantize_compare_multi(ctypes.cast(arr, ctypes.c_void_p), ctypes.cast(ref_arr, ctypes.c_void_p), n,
                                         _p(results[0]), _p(results[1]), ctypes.c_void_p(_stream(dev)))
    _check(st, "mx_quantize_compare_multi")
    return outs, results[0, :2 * n], results[1, :2 * n]


def grid_equal_multi(pairs, out=None):
    """mx_grid_equal_multi over a list of (a, b) CUDA tensor pairs. Returns (mismatches, first_index):
    int64 device tensors of len(pairs) entries (no host synchronisation)."""
    n = len(pairs)
    dev = pairs[0][0].device if pairs else torch.device("cuda")
    if out is None:
        out = torch.empty((2, max(n, 1)), dtype=torch.int64, device=dev)
    arr = compare_pair_array(pairs)
    st = lib().mx_grid_equal_multi(ctypes.cast(arr, ctypes.c_void_p), n, _p(out[0]), _p(out[1]),
                                   ctypes.c_void_p(_stream(dev)))
    _check(st, "mx_grid_equal_multi")
    return out[0, :n], out[1, :n]


def swizzle_scales(s: torch.Tensor, group_rows=None, out=None):
    """mx_swizzle_scales on raw scales [rows, kblocks] (uint8, CUDA)."""
    assert s.dtype == torch.uint8 and s.dim() == 2 and s.is_contiguous()
    rows, kb = s.shape
    if group_rows is not None:
        gr = np.ascontiguousarray(np.asarray(group_rows, dtype=np.int64))       # host memory, read during the call
        gptr, ng = ctypes.c_void_p(gr.ctypes.data), int(gr.size)
    else:
        gr, gptr, ng = None, None, 0
    if out is None:
        size = grouped_swizzled_scale_bytes(gr, kb) if gr is not None else swizzled_scale_bytes(rows, kb)
        out = torch.empty(size, dtype=torch.uint8, device=s.device)
    st = lib().mx_swizzle_scales(_p(s), rows, kb, gptr, ng, _p(out), ctypes.c_void_p(_stream(s.device)))
    _check(st, "mx_swizzle_scales")
    return out


def _out_code(dtype) -> int:
    return {torch.float32: MX_OUT_F32, torch.bfloat16: MX_OUT_BF16}[dtype]


def gemm(qa, sa_swz, qb, sb_swz, out_dtype=torch.bfloat16, out=None):
    """mx_gemm: C[M, N] = A . B^T from K-major E4M3 operands and tensor-core-layout scales."""
    M, K = qa.shape
    N = qb.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=qa.device)
    st = lib().mx_gemm(_p(qa), _p(sa_swz), _p(qb), _p(sb_swz), M, N, K, _p(out), out.stride(0),
                       _out_code(out.dtype), ctypes.c_void_p(_stream(qa.device)))
    _check(st, "mx_gemm")
    return out


def grouped_gemm(qa, sa_swz, qb, sb_swz, row_offsets, out_dtype=torch.bfloat16, out=None):
    """mx_grouped_gemm: rows [off[g], off[g+1]) of A against qb[g]. row_offsets: int32 CUDA [G+1]."""
    total, K = qa.shape
    G, N, K2 = qb.shape
    assert K2 == K and row_offsets.dtype == torch.int32 and row_offsets.numel() == G + 1
    if out is None:
        out = torch.empty((total, N), dtype=out_dtype, device=qa.device)
    st = lib().mx_grouped_gemm(_p(qa), _p(sa_swz), _p(qb), _p(sb_swz), _p(row_offsets), G, total, N, K, _p(out),
                               out.stride(0), _out_code(out.dtype), ctypes.c_void_p(_stream(qa.device)))
    _check(st, "mx_grouped_gemm")
    return out


def grouped_gemm_swiglu_quant(qa, sa_swz, qb, sb_swz, row_offsets, group_rows, out=None):
    """mx_grouped_gemm_swiglu_quant. qb: [G, 2 n, K] with gate/up rows interleaved per 128;
    group_rows: rows per expert (host), for the size of h's grouped scale layout. Returns
    (h_q uint8 [total, n], h_s uint8 grouped tensor-core layout of [total, n / 32])."""
    total, K = qa.shape
    G, N2, K2 = qb.shape
    assert K2 == K and N2 % 2 == 0 and row_offsets.dtype == torch.int32 and row_offsets.numel() == G + 1
    n = N2 // 2
    if out is None:
        u8 = dict(dtype=torch.uint8, device=qa.device)
        out = (torch.empty((total, n), **u8),
               torch.empty(grouped_swizzled_scale_bytes([int(r) for r in group_rows], n // 32), **u8))
    hq, hs = out
    st = lib().mx_grouped_gemm_swiglu_quant(_p(qa), _p(sa_swz), _p(qb), _p(sb_swz), _p(row_offsets), G, total, n,
                                            K, _p(hq), _p(hs), ctypes.c_void_p(_stream(qa.device)))
    _check(st, "mx_grouped_gemm_swiglu_quant")
    return hq, hs


def quantize_block128(x: torch.Tensor, pow2_scales: bool, out=None):
    """mx_quantize_block128 on a 2-D BF16 CUDA tensor: FP8 blockwise codes with one FP32
    (pow2_scales=False) or power-of-two (pow2_scales=True) scale per 128 x 128 block.
    Returns (q uint8 [M, K], scales float32 [ceil(M/128), ceil(K/128)])."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    M, K = x.shape
    if out is None:
        out = (torch.empty((M, K), dtype=torch.uint8, device=x.device),
               torch.empty(((M + 127) // 128, (K + 127) // 128), dtype=torch.float32, device=x.device))
    q, sc = out
    st = lib().mx_quantize_block128(_p(x), M, K, x.stride(0), 1 if pow2_scales else 0, _p(q), _p(sc),
                                    ctypes.c_void_p(_stream(x.device)))
    _check(st, "mx_quantize_block128")
    return q, sc


def grid_equal(a: torch.Tensor, b: torch.Tensor, out=None):
    """mx_grid_equal over the bytes of two CUDA tensors. Returns (mismatches, first_index) as
    1-element int64 device tensors (no host synchronisation)."""
    assert a.is_contiguous() and b.is_contiguous()
    n = a.numel() * a.element_size()
    assert b.numel() * b.element_size() == n
    if out is None:
        out = torch.empty(2, dtype=torch.int64, device=a.device)
    cnt, first = out[0:1], out[1:2]
    st = lib().mx_grid_equal(_p(a), _p(b), n, _p(cnt), _p(first), ctypes.c_void_p(_stream(a.device)))
    _check(st, "mx_grid_equal")
    return cnt, first


def device_error() -> int:
    """Reads and clears the device status word (synchronizes). 0 means no error bit set."""
    bits = ctypes.c_uint32(0)
    st = lib().mx_device_error(ctypes.byref(bits))
    if st not in (0, -6):
        _check(st, "mx_device_error")
    return int(bits.value)


def set_wait_timeout_ns(ns: int):
    lib().mx_set_wait_timeout_ns(int(ns))


GEMM_PAIR, GEMM_SINGLE = 0, 1


def set_gemm_variant(variant: int):
    """0: CTA-pair GEMM kernel (default); 1: single-CTA kernel."""
    lib().mx_set_gemm_variant(int(variant))


QUANT_REGISTERS, QUANT_TMA, QUANT_SPLIT = 0, 1, 2


def set_quantize_variant(variant: int):
    """0: register-staged quantizer (default; split loads for long rowwise tile walks); 1: TMA-staged
    quantizer; 2: register-staged with split loads for every rowwise call. Same bytes in every case."""
    lib().mx_set_quantize_variant(int(variant))
