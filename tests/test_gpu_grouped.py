"""GPU parity: mx_swizzle_scales (single and grouped) bit-exact, and mx_grouped_gemm against the
fp64 oracle within the GEMM tolerance."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_gemm_close, to_np
from mxfp8_block_scaled_07_b200 import mx, synth

pytestmark = pytest.mark.gpu


# kb % 16 == 0 takes the 16-byte-load kernel, kb % 4 == 0 the 32-bit-load one, the rest byte loads.
@pytest.mark.parametrize("rows,kb", [(1, 1), (128, 4), (300, 13), (1024, 64), (4097, 130), (1000, 24), (513, 32),
                                     (777, 48)])
def test_swizzle_single_group(rows, kb):
    s = synth.random_bytes(rows * kb, seed=rows + kb).reshape(rows, kb)
    out = mx.swizzle_scales(s.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(to_np(out), oracle.swizzle(s.numpy()))


@pytest.mark.parametrize("offset", [1, 4])
def test_swizzle_unaligned_source(offset):
    """A raw-scale pointer that is not 16-byte (or not 4-byte) aligned takes the narrower loads."""
    rows, kb = 300, 64
    s = synth.random_bytes(rows * kb, seed=9).reshape(rows, kb)
    buf = torch.zeros(rows * kb + 16, dtype=torch.uint8, device="cuda")
    buf[offset:offset + rows * kb] = s.reshape(-1).cuda()
    out = mx.swizzle_scales(buf[offset:offset + rows * kb].view(rows, kb))
    torch.cuda.synchronize()
    assert np.array_equal(to_np(out), oracle.swizzle(s.numpy()))


@pytest.mark.parametrize("groups,kb", [([0, 5, 128, 129, 300, 0, 1], 64), ([7] * 200, 64), ([0], 64),
                                       ([256, 0, 0, 3], 64), ([0, 5, 128, 129, 300, 0, 1], 24),
                                       ([130, 0, 1, 255], 13)])
def test_swizzle_grouped(groups, kb):
    rows = sum(groups)
    s = synth.random_bytes(max(rows, 1) * kb, seed=len(groups))[: rows * kb].reshape(rows, kb)
    if rows == 0:
        pytest.skip("no rows")
    out = mx.swizzle_scales(s.cuda(), groups)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(out), oracle.swizzle(s.numpy(), groups))


def grouped_case(counts, N, K, out_dtype, seed=0, device_inputs=None):
    counts = [int(c) for c in counts]
    off = synth.group_offsets(counts)
    G = len(counts)
    rows = off[-1]
    if device_inputs is None:
        X = synth.normal_bf16((rows, K), seed=seed, outlier_frac=0.01, outlier_scale=100.0)
        W = synth.normal_bf16((G, N, K), std=0.02, seed=seed + 1)
    else:
        X, W = device_inputs
    Xd, Wd = X.cuda(), W.cuda()
    qx, sx_raw, _, _ = mx.quantize(Xd, True, False, swizzle=False)
    sx = mx.swizzle_scales(sx_raw, counts)
    qw, sw, _, _ = mx.quantize(Wd.reshape(G * N, K), True, False, swizzle=True)
    if N % 128:
        # B's scales are G consecutive per-expert layouts, each padded to 128 rows on its own; one
        # layout of all G * N rows matches that only when N is a multiple of 128.
        sw = torch.cat([mx.quantize(Wd[g].contiguous(), True, False, swizzle=True)[1] for g in range(G)])
    offs = torch.tensor(off, dtype=torch.int32, device="cuda")
    c = mx.grouped_gemm(qx, sx, qw.reshape(G, N, K), sw, offs, out_dtype=out_dtype)
    torch.cuda.synchronize()
    return X, W, off, c


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_grouped_small_ragged_with_empty_groups(out_dtype, grouped_variant):
    counts = [0, 5, 128, 129, 300, 0, 1, 64, 256, 257, 511, 2]
    N, K = 384, 256
    X, W, off, c = grouped_case(counts, N, K, out_dtype, seed=3)
    qx, sx = oracle.quantize_rowwise(X)
    qw, sw = oracle.quantize_rowwise(W.reshape(-1, K))
    ref, abs_sum = oracle.grouped_gemm(qx, sx, qw.reshape(len(counts), N, K), sw.reshape(len(counts), N, K // 32), off)
    assert_gemm_close(to_np(c.float()), ref, abs_sum, out_dtype == torch.bfloat16, "grouped small")


def test_grouped_bad_offsets_set_device_error_and_write_nothing(grouped_variant):
    counts = [64, 64]
    N, K = 256, 128
    X = synth.normal_bf16((128, K), seed=1).cuda()
    W = synth.normal_bf16((2, N, K), seed=2).cuda()
    qx, sx_raw, _, _ = mx.quantize(X, True, False, swizzle=False)
    sx = mx.swizzle_scales(sx_raw, counts)
    qw, sw, _, _ = mx.quantize(W.reshape(2 * N, K), True, False, swizzle=True)
    mx.device_error()
    bad = torch.tensor([0, 100, 64], dtype=torch.int32, device="cuda")      # decreasing, wrong total
    out = torch.full((128, N), 3.0, device="cuda")
    mx.grouped_gemm(qx, sx, qw.reshape(2, N, K), sw, bad, out=out)
    assert mx.device_error() == 2
    assert torch.all(out == 3.0)


def test_moe_layer_full_size_sampled():
    """Qwen3-30B-A3B MoE layer at full size: 163 840 routed rows (Zipf(1.1) top-8 over 128 experts),
    gate_up (N 1536, K 2048) and down (N 2048, K 768), BF16 out; sampled rows of every expert."""
    counts, Xp, H, W1, W2 = synth.moe_inputs(device="cuda")
    counts = [int(c) for c in counts]
    off = synth.group_offsets(counts)
    G = len(counts)
    g = np.random.default_rng(4)
    for name, X, W in (("gate_up", Xp, W1), ("down", H, W2)):
        N, K = W.shape[1], W.shape[2]
        _, _, _, c = grouped_case(counts, N, K, torch.bfloat16, device_inputs=(X, W))
        for e in range(G):
            if counts[e] == 0:
                continue
            rr = np.unique(np.concatenate([[off[e], off[e + 1] - 1], off[e] + g.integers(0, counts[e], 2)]))
            qa, sa = oracle.quantize_rowwise(X[torch.from_numpy(rr).cuda()].cpu())
            cols = np.unique(g.integers(0, N, 96))
            qb, sb = oracle.quantize_rowwise(W[e][torch.from_numpy(cols).cuda()].cpu())
            ref, abs_sum = oracle.gemm(qa, sa, qb, sb)
            assert_gemm_close(to_np(c[torch.from_numpy(rr).cuda()][:, torch.from_numpy(cols).cuda()].float()),
                              ref, abs_sum, True, f"{name} expert {e}")


@pytest.mark.parametrize("K,N", [(32, 200), (128, 640), (384, 200), (768, 200), (768, 640), (896, 128)])
def test_grouped_short_k_shapes(K, N, grouped_variant):
    """Short K (1 to 7 k-blocks of 128, the MoE down projection's 768 among them) with N not a
    multiple of 128 and experts of 0, 1, 128, 255, 256 and 300 rows."""
    counts = [128, 0, 1, 300, 255, 256, 3]
    X, W, off, c = grouped_case(counts, N, K, torch.float32, seed=K + N)
    qx, sx = oracle.quantize_rowwise(X)
    qw, sw = oracle.quantize_rowwise(W.reshape(-1, K))
    G = len(counts)
    ref, abs_sum = oracle.grouped_gemm(qx, sx, qw.reshape(G, N, K), sw.reshape(G, N, K // 32), off)
    assert_gemm_close(to_np(c), ref, abs_sum, False, f"grouped K={K} N={N}")


def test_grouped_many_units_per_pair():
    """More 256-row tiles per expert than one, across many experts of up to 700 rows, K = 768."""
    g = np.random.default_rng(11)
    counts = [int(c) for c in g.integers(0, 600, 24)]
    N, K = 384, 768
    X, W, off, c = grouped_case(counts, N, K, torch.bfloat16, seed=5)
    qx, sx = oracle.quantize_rowwise(X)
    qw, sw = oracle.quantize_rowwise(W.reshape(-1, K))
    G = len(counts)
    ref, abs_sum = oracle.grouped_gemm(qx, sx, qw.reshape(G, N, K), sw.reshape(G, N, K // 32), off)
    assert_gemm_close(to_np(c.float()), ref, abs_sum, True, "grouped many units")


def test_expired_waits_end_the_grouped_gemm_cleanly(grouped_variant):
    """With a 1 ns deadline every wait that does not succeed at once expires: the grouped kernel
    records error bit 1, drains its copies and MMAs and returns; the next grouped GEMM is exact. A
    wait's first try may itself block for a while (the hardware's suspend window), so K is long
    enough for the tiles to outlast it, and the launch is repeated until a wait has expired."""
    expired_waits_case(8192)


def expired_waits_case(K):
    g = np.random.default_rng(12)
    counts = [int(c) for c in g.integers(0, 2000, 40)]
    G, N = len(counts), 1024
    X = synth.normal_bf16((sum(counts), K), seed=6).cuda()
    W = synth.normal_bf16((G, N, K), std=0.02, seed=7).cuda()
    qx, sx_raw, _, _ = mx.quantize(X, True, False, swizzle=False)
    sx = mx.swizzle_scales(sx_raw, counts)
    qw, sw, _, _ = mx.quantize(W.reshape(G * N, K), True, False, swizzle=True)
    offs = torch.tensor(synth.group_offsets(counts), dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    assert mx.device_error() == 0
    mx.set_wait_timeout_ns(1)
    try:
        for _ in range(8):
            mx.grouped_gemm(qx, sx, qw.reshape(G, N, K), sw, offs, out_dtype=torch.bfloat16)
            torch.cuda.synchronize()
            bits = mx.device_error()
            if bits:
                break
    finally:
        mx.set_wait_timeout_ns(0)
    assert bits == 1
    counts = [3, 0, 300, 129]
    X, W, off, c = grouped_case(counts, 256, 384, torch.float32, seed=7)
    qx, sx = oracle.quantize_rowwise(X)
    qw, sw = oracle.quantize_rowwise(W.reshape(-1, 384))
    ref, abs_sum = oracle.grouped_gemm(qx, sx, qw.reshape(4, 256, 384), sw.reshape(4, 256, 384 // 32), off)
    assert_gemm_close(to_np(c), ref, abs_sum, False, "grouped after expired waits")
    assert mx.device_error() == 0


def test_library_cross_check_scaled_grouped_mm_blockwise_1x32():
    """torch's grouped MXFP8 GEMM (scaled_grouped_mm, BlockWise1x32 + SWIZZLE_32_4_4) fed with this
    library's bytes, A's grouped scale layout (each expert padded to 128 rows) and B's per-expert
    layouts must agree with the oracle as well: an independent consumer of the grouped layout."""
    import torch.nn.functional as F

    counts = [0, 5, 128, 129, 300, 0, 1, 64, 256, 257]
    N, K = 256, 384
    X, W, off, c = grouped_case(counts, N, K, torch.bfloat16, seed=21)
    G = len(counts)
    Xd, Wd = X.cuda(), W.cuda()
    qx, sx_raw, _, _ = mx.quantize(Xd, True, False, swizzle=False)
    sx = mx.swizzle_scales(sx_raw, counts)
    qw, sw, _, _ = mx.quantize(Wd.reshape(G * N, K), True, False, swizzle=True)
    kb_pad = (K // 32 + 3) // 4 * 4
    ends = torch.tensor(off[1:], dtype=torch.int32, device="cuda")
    try:
        lib = F.scaled_grouped_mm(qx.view(torch.float8_e4m3fn),
                                  qw.view(torch.float8_e4m3fn).reshape(G, N, K).transpose(-2, -1),
                                  sx.view(torch.float8_e8m0fnu).reshape(-1, kb_pad), F.ScalingType.BlockWise1x32,
                                  sw.view(torch.float8_e8m0fnu).reshape(G, -1), F.ScalingType.BlockWise1x32,
                                  swizzle_a=F.SwizzleType.SWIZZLE_32_4_4, swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                                  offs=ends, output_dtype=torch.bfloat16)
    except (RuntimeError, TypeError, NotImplementedError, AttributeError) as e:  # pragma: no cover
        pytest.skip(f"torch scaled_grouped_mm MXFP8 path unavailable: {e}")
    torch.cuda.synchronize()
    qxo, sxo = oracle.quantize_rowwise(X)
    qwo, swo = oracle.quantize_rowwise(W.reshape(-1, K))
    ref, abs_sum = oracle.grouped_gemm(qxo, sxo, qwo.reshape(G, N, K), swo.reshape(G, N, K // 32), off)
    assert_gemm_close(to_np(lib.float()), ref, abs_sum, True, "torch scaled_grouped_mm on our layouts")
    assert_gemm_close(to_np(c.float()), ref, abs_sum, True, "mx_grouped_gemm")
