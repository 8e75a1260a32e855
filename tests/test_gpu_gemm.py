"""GPU parity: mx_gemm against the fp64 oracle, elementwise within
|c - ref| <= 1e-5 * sum_k |a_k b_k| (+ 2^-8 |ref| for BF16 output).

Operands are quantized by the oracle from the seeded BF16 inputs (the oracle never sees a GPU
result); the GPU quantizes the same inputs itself and the bytes are first checked equal."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_gemm_close, to_np
from mxfp8_block_scaled_07_b200 import mx, synth

pytestmark = pytest.mark.gpu


def gpu_operand(x: torch.Tensor):
    """Rowwise quantization on the GPU with the tensor-core scale layout."""
    q, s, _, _ = mx.quantize(x, True, False, swizzle=True)
    return q, s


def check_case(A, B, out_dtype, what):
    qa_o, sa_o = oracle.quantize_rowwise(A)
    qb_o, sb_o = oracle.quantize_rowwise(B)
    ref, abs_sum = oracle.gemm(qa_o, sa_o, qb_o, sb_o)
    qa, sa = gpu_operand(A.cuda())
    qb, sb = gpu_operand(B.cuda())
    c = mx.gemm(qa, sa, qb, sb, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(qa), qa_o) and np.array_equal(to_np(qb), qb_o)
    return assert_gemm_close(to_np(c.float()), ref, abs_sum, out_dtype == torch.bfloat16, what)


def test_pr1_full_fp32(gemm_variant):
    A, B = synth.pr1_inputs()
    check_case(A, B, torch.float32, "PR1 256x128x512")


@pytest.mark.parametrize("mnk", [(1, 1, 32), (128, 256, 128), (130, 300, 160), (256, 512, 1024), (129, 257, 4160),
                                 (384, 768, 544), (77, 136, 2048), (520, 1024, 256), (1000, 600, 640)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_ragged_shapes(mnk, out_dtype, gemm_variant):
    M, N, K = mnk
    A = synth.normal_bf16((M, K), seed=M + 3, outlier_frac=0.01, outlier_scale=100.0)
    B = synth.normal_bf16((N, K), std=0.02, seed=N + 5, outlier_frac=0.001, outlier_scale=50.0)
    check_case(A, B, out_dtype, f"{M}x{N}x{K}")


def test_identity_like_b_selects_columns_of_a(gemm_variant):
    # B = rows of the identity (scaled by powers of two) picks single K-columns of A exactly.
    M, K = 160, 256
    A = synth.normal_bf16((M, K), seed=11)
    N = 64
    B = torch.zeros((N, K), dtype=torch.bfloat16)
    cols = np.random.default_rng(3).choice(K, N, replace=False)
    for n, k in enumerate(cols):
        B[n, k] = 2.0 ** (n % 7 - 3)
    qa_o, sa_o = oracle.quantize_rowwise(A)
    c = mx.gemm(*gpu_operand(A.cuda()), *gpu_operand(B.cuda()), out_dtype=torch.float32)
    dq = oracle.dequantize(qa_o, sa_o)
    expect = dq[:, cols] * (2.0 ** (np.arange(N) % 7 - 3))[None, :]
    assert np.array_equal(to_np(c).astype(np.float64), expect)


def test_out_leading_dimension_and_untouched_padding(gemm_variant):
    M, N, K = 200, 264, 320
    A = synth.normal_bf16((M, K), seed=21)
    B = synth.normal_bf16((N, K), seed=22)
    qa, sa = gpu_operand(A.cuda())
    qb, sb = gpu_operand(B.cuda())
    big = torch.full((M + 3, N + 40), 7.0, dtype=torch.bfloat16, device="cuda")
    out = big[:M, :N]
    mx.gemm(qa, sa, qb, sb, out=out)
    ref = mx.gemm(qa, sa, qb, sb, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    assert torch.all(big[:, N:] == 7.0) and torch.all(big[M:, :] == 7.0)


def test_library_cross_check_scaled_mm_blockwise_1x32():
    """torch's cuBLAS MXFP8 path (BlockWise1x32 + SWIZZLE_32_4_4) on our quantized bytes and swizzled
    scales must agree with the oracle too: a check of the scale layout by an independent consumer."""
    import torch.nn.functional as F

    M, N, K = 256, 384, 512
    A = synth.normal_bf16((M, K), seed=31, outlier_frac=0.01, outlier_scale=100.0)
    B = synth.normal_bf16((N, K), seed=32)
    qa, sa = gpu_operand(A.cuda())
    qb, sb = gpu_operand(B.cuda())
    try:
        ref_lib = F.scaled_mm(qa.view(torch.float8_e4m3fn), qb.view(torch.float8_e4m3fn).t(),
                              sa.view(torch.float8_e8m0fnu), F.ScalingType.BlockWise1x32,
                              sb.view(torch.float8_e8m0fnu), F.ScalingType.BlockWise1x32,
                              swizzle_a=F.SwizzleType.SWIZZLE_32_4_4, swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                              output_dtype=torch.float32)
    except (RuntimeError, TypeError, NotImplementedError) as e:  # pragma: no cover
        pytest.skip(f"torch scaled_mm MXFP8 path unavailable: {e}")
    qa_o, sa_o = oracle.quantize_rowwise(A)
    qb_o, sb_o = oracle.quantize_rowwise(B)
    ref, abs_sum = oracle.gemm(qa_o, sa_o, qb_o, sb_o)
    assert_gemm_close(to_np(ref_lib), ref, abs_sum, False, "torch scaled_mm on our layout")
    ours = mx.gemm(qa, sa, qb, sb, out_dtype=torch.float32)
    assert_gemm_close(to_np(ours), ref, abs_sum, False, "mx_gemm")


def sampled_check(a_rows, b_rows, c_dev, rows, cols, n_rand, bf16, what, seed=0):
    """Checks full rows `rows`, full columns `cols` and an n_rand x n_rand grid of random elements
    of C = quant(A) . quant(B)^T. a_rows(idx) / b_rows(idx) return the BF16 operand rows (the
    contraction dimension contiguous) as CPU tensors; the oracle quantizes them itself."""
    g = np.random.default_rng(seed)
    M, N = c_dev.shape
    C = to_np(c_dev.float())
    qA, sA = oracle.quantize_rowwise(a_rows(np.arange(M)))
    qB, sB = oracle.quantize_rowwise(b_rows(np.arange(N)))
    worst = 0.0
    ref, abs_sum = oracle.gemm(qA[rows], sA[rows], qB, sB)
    worst = max(worst, assert_gemm_close(C[rows], ref, abs_sum, bf16, what + " rows"))
    ref, abs_sum = oracle.gemm(qA, sA, qB[cols], sB[cols])
    worst = max(worst, assert_gemm_close(C[:, cols], ref, abs_sum, bf16, what + " cols"))
    rr = np.unique(g.integers(0, M, n_rand))
    cc = np.unique(g.integers(0, N, n_rand))
    ref, abs_sum = oracle.gemm(qA[rr], sA[rr], qB[cc], sB[cc])
    worst = max(worst, assert_gemm_close(C[np.ix_(rr, cc)], ref, abs_sum, bf16, what + " elements"))
    return worst


def rows_of(t_dev):
    """Row provider for a CUDA tensor whose rows are operand rows."""
    return lambda idx: t_dev[torch.from_numpy(np.asarray(idx)).to(t_dev.device)].cpu()


def cols_of(t_dev):
    """Row provider for the transpose of a CUDA tensor (operand rows are its columns)."""
    return lambda idx: t_dev[:, torch.from_numpy(np.asarray(idx)).to(t_dev.device)].t().contiguous().cpu()


@pytest.mark.parametrize("M", synth.FWD_TOKENS)
def test_fwd_linear_full_size_sampled(M):
    # Qwen3-8B forward linear: X[M, 4096] (lognormal channels) . W_gate_up[24576, 4096]^T, BF16 out.
    X = synth.fwd_activations(M, device="cuda")
    W = synth.sync_weight(0, 2, device="cuda")
    qx, sx = gpu_operand(X)
    qw, sw = gpu_operand(W)
    c = mx.gemm(qx, sx, qw, sw, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    sampled_check(rows_of(X), rows_of(W), c, np.array([0, M - 1]), np.array([0, 24575]), 64, True, f"fwd M={M}")


def test_update_step_full_size_sampled():
    """Qwen3-8B update micro-batch of 12288 tokens: fprop Y = X W^T, dgrad dX = dY W, wgrad
    dW = dY^T X, with the transposed operands from the fused row+col quantizer."""
    X, W, dY = synth.update_inputs(device="cuda")
    qx_r, sx_r, qx_c, sx_c = mx.quantize(X, True, True)
    qw_r, sw_r, qw_c, sw_c = mx.quantize(W, True, True)
    qd_r, sd_r, qd_c, sd_c = mx.quantize(dY, True, True)
    Y = mx.gemm(qx_r, sx_r, qw_r, sw_r)           # [12288 tokens, 12288 out]
    dX = mx.gemm(qd_r, sd_r, qw_c, sw_c)          # [12288 tokens, 4096 hidden], K = 12288 out
    dW = mx.gemm(qd_c, sd_c, qx_c, sx_c)          # [12288 out, 4096 hidden], K = 12288 tokens
    torch.cuda.synchronize()
    sampled_check(rows_of(X), rows_of(W), Y, np.array([5, 12287]), np.array([0, 12287]), 48, True, "fprop")
    sampled_check(rows_of(dY), cols_of(W), dX, np.array([0, 9000]), np.array([17, 4095]), 48, True, "dgrad")
    sampled_check(cols_of(dY), cols_of(X), dW, np.array([1, 12287]), np.array([0, 4095]), 48, True, "wgrad")


def test_update_step_fp32_out_long_k():
    """The update step's K = 12 288 contractions (dgrad over the output features, wgrad over the
    tokens) with fp32 output, where the 2^-8 term of the BF16 bound cannot hide the accumulator:
    every sampled element within 1e-5 * sum_k |a_k b_k| of the fp64 oracle. Also the forward
    K = 4096 product in fp32. Prints the worst err / sum|ab| seen."""
    X, W, dY = synth.update_inputs(device="cuda")
    _, _, qx_c, sx_c = mx.quantize(X, False, True)
    qw_r, sw_r, qw_c, sw_c = mx.quantize(W, True, True)
    qd_r, sd_r, qd_c, sd_c = mx.quantize(dY, True, True)
    qx_r, sx_r, _, _ = mx.quantize(X, True, False)
    dX = mx.gemm(qd_r, sd_r, qw_c, sw_c, out_dtype=torch.float32)      # K = 12288
    dW = mx.gemm(qd_c, sd_c, qx_c, sx_c, out_dtype=torch.float32)      # K = 12288
    Y = mx.gemm(qx_r, sx_r, qw_r, sw_r, out_dtype=torch.float32)       # K = 4096
    torch.cuda.synchronize()
    worst = {
        "dgrad": sampled_check(rows_of(dY), cols_of(W), dX, np.array([3, 12287]), np.array([0, 4095]), 48, False,
                               "dgrad fp32", seed=1),
        "wgrad": sampled_check(cols_of(dY), cols_of(X), dW, np.array([0, 12287]), np.array([1, 4095]), 48, False,
                               "wgrad fp32", seed=2),
        "fprop": sampled_check(rows_of(X), rows_of(W), Y, np.array([0, 12287]), np.array([7, 12287]), 48, False,
                               "fprop fp32", seed=3),
    }
    print("worst |c - ref| / sum|ab| (bound 1e-5):", {k: f"{v:.3e}" for k, v in worst.items()})
    assert max(worst.values()) <= 1e-5


def test_expired_waits_end_the_gemm_cleanly(gemm_variant):
    """With a 1 ns deadline every wait that does not succeed at once expires: the kernel records
    error bit 1, every role stops, in-flight copies and MMAs are drained (those drain waits keep a
    floor of 1 s), TMEM is freed and the launch returns. The context stays usable: the next GEMM
    under the default deadline is exact."""
    M, N, K = 1024, 1024, 16384
    A = synth.normal_bf16((M, K), seed=91)
    B = synth.normal_bf16((N, K), seed=92)
    qa, sa = gpu_operand(A.cuda())
    qb, sb = gpu_operand(B.cuda())
    torch.cuda.synchronize()
    assert mx.device_error() == 0
    mx.set_wait_timeout_ns(1)
    try:
        mx.gemm(qa, sa, qb, sb, out_dtype=torch.float32)
        torch.cuda.synchronize()
        bits = mx.device_error()
    finally:
        mx.set_wait_timeout_ns(0)
    assert bits == 1
    check_case(A[:256, :1024].contiguous(), B[:384, :1024].contiguous(), torch.float32, "after expired waits")
    assert mx.device_error() == 0
