"""Shared test helpers (no method arithmetic beyond what the oracle provides)."""
import numpy as np
import torch

import oracle


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def scale_positions(rows: int, kblocks: int, group_rows=None) -> np.ndarray:
    """Byte position of every raw scale (r, c) inside the tensor-core layout, obtained by
    swizzling tag planes with the oracle: int64 [rows, kblocks]."""
    tag = np.arange(rows * kblocks, dtype=np.int64).reshape(rows, kblocks)
    pos = np.zeros(oracle.swizzled_size(rows, kblocks, group_rows), np.int64)
    for plane in range(4):
        part = ((tag >> (8 * plane)) & 0xFF).astype(np.uint8)
        pos |= oracle.swizzle(part, group_rows).astype(np.int64) << (8 * plane)
    filled = oracle.swizzle(np.ones((rows, kblocks), np.uint8), group_rows).astype(bool)
    out = np.empty(rows * kblocks, np.int64)
    out[pos[filled]] = np.nonzero(filled)[0]
    return out.reshape(rows, kblocks)


def assert_gemm_close(c_gpu, ref, abs_sum, bf16: bool, what=""):
    """|c - ref| <= 1e-5 * sum_k |a_k b_k| (+ 2^-8 |ref| for BF16 output), elementwise."""
    c = np.asarray(c_gpu, np.float64)
    bound = 1e-5 * abs_sum + (2.0 ** -8 * np.abs(ref) if bf16 else 0.0)
    err = np.abs(c - ref)
    bad = ~(err <= bound)
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(
            f"{what}: {bad.sum()} of {bad.size} outside tolerance; first at {tuple(i)}: gpu {c[tuple(i)]!r} "
            f"ref {ref[tuple(i)]!r} bound {bound[tuple(i)] if np.ndim(bound) else bound!r}")
    ratio = np.where(abs_sum > 0, err / np.maximum(abs_sum, 1e-300), 0.0)
    return float(ratio.max()) if ratio.size else 0.0


def check_sampled_rows(x_dev: torch.Tensor, q_dev: torch.Tensor, s_dev: torch.Tensor, rows, group_rows=None,
                       swizzled: bool = True, what: str = ""):
    """Rowwise quantization of the CUDA tensor x_dev, checked against the oracle on the sampled
    rows: E4M3 codes, and the scale bytes either raw ([rows, K/32]) or at their positions in the
    (grouped) tensor-core layout, whose pad bytes must all be 0. The oracle quantizes the BF16 rows
    itself; nothing of the GPU result reaches it."""
    rows = np.unique(np.asarray(rows, np.int64))
    M, K = x_dev.shape
    r_dev = torch.from_numpy(rows).to(x_dev.device)
    qo, so = oracle.quantize_rowwise(x_dev[r_dev].cpu())
    q = to_np(q_dev[r_dev])
    bad = np.argwhere(q != qo)
    assert bad.size == 0, f"{what}: {len(bad)} code bytes differ; first at row {rows[bad[0][0]]} col {bad[0][1]}"
    s_np = to_np(s_dev)
    if not swizzled:
        assert np.array_equal(s_np[rows], so), f"{what}: raw scales"
        return
    pos = scale_positions(M, K // 32, group_rows)
    assert np.array_equal(s_np.reshape(-1)[pos[rows]], so), f"{what}: scale bytes in the layout"
    pad = np.ones(s_np.size, bool)
    pad[pos.reshape(-1)] = False
    assert not s_np.reshape(-1)[pad].any(), f"{what}: nonzero pad bytes in the scale layout"
