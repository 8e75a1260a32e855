"""GPU parity: mx_quantize (rowwise / columnwise, raw / tensor-core scale layout) against the CPU
oracle, bit for bit, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from helpers import scale_positions, to_np
from mxfp8_block_scaled_07_b200 import mx, synth

pytestmark = pytest.mark.gpu


def run_both(x_cpu: torch.Tensor, rowwise=True, colwise=False, ld_pad=0):
    """Quantize on the GPU (raw and swizzled) and with the oracle; assert every byte agrees."""
    M, K = x_cpu.shape
    if ld_pad:
        big = torch.zeros((M, K + ld_pad), dtype=torch.bfloat16)
        big[:, :K] = x_cpu
        xg = big.cuda()[:, :K]
    else:
        xg = x_cpu.cuda()
    raw = mx.quantize(xg, rowwise, colwise, swizzle=False)
    swz = mx.quantize(xg, rowwise, colwise, swizzle=True)
    torch.cuda.synchronize()
    if rowwise:
        q, s = oracle.quantize_rowwise(x_cpu)
        assert np.array_equal(to_np(raw[0]), q), "rowwise elements (raw-scale call)"
        assert np.array_equal(to_np(swz[0]), q), "rowwise elements (swizzled call)"
        assert np.array_equal(to_np(raw[1]), s), "rowwise raw scales"
        assert np.array_equal(to_np(swz[1]), oracle.swizzle(s)), "rowwise swizzled scales"
    if colwise:
        qT, sT = oracle.quantize_colwise(x_cpu)
        assert np.array_equal(to_np(raw[2]), qT), "colwise elements"
        assert np.array_equal(to_np(swz[2]), qT), "colwise elements (swizzled call)"
        assert np.array_equal(to_np(raw[3]), sT), "colwise raw scales"
        assert np.array_equal(to_np(swz[3]), oracle.swizzle(sT)), "colwise swizzled scales"


def test_pr1_operands_row_and_col(quant_variant):
    A, B = synth.pr1_inputs()
    run_both(A, True, True)
    run_both(B, True, True)


@pytest.mark.parametrize("shape", [(1, 32), (33, 96), (130, 160), (256, 512), (300, 1056), (7, 4096), (129, 4128)])
def test_rowwise_ragged_shapes(shape, quant_variant):
    x = synth.normal_bf16(shape, std=0.5, seed=shape[0] * 7 + shape[1], outlier_frac=0.01, outlier_scale=100.0)
    run_both(x, True, False)


@pytest.mark.parametrize("shape", [(32, 32), (64, 96), (160, 288), (384, 544), (96, 4096), (4096, 160)])
def test_row_and_col_ragged_shapes(shape, quant_variant):
    x = synth.normal_bf16(shape, std=3.0, seed=shape[0] + shape[1], outlier_frac=0.01, outlier_scale=50.0)
    run_both(x, True, True)
    run_both(x, False, True)


def test_strided_input(quant_variant):
    x = synth.normal_bf16((200, 320), seed=4)
    run_both(x, True, False, ld_pad=24)
    x = synth.normal_bf16((192, 320), seed=5)
    run_both(x, True, True, ld_pad=8)


@pytest.mark.parametrize("seed", [0, 1])
def test_special_values_nan_inf_zero_subnormal(seed, quant_variant):
    x = synth.special_bf16((256, 1024), seed=seed)
    run_both(x, True, True)


def test_every_bf16_pattern_in_blocks(quant_variant):
    # All 65536 BF16 bit patterns, 32 to a block, in two arrangements (sorted: blocks of nearby
    # magnitude; shuffled: mixed magnitudes, so most elements sit far below their block's amax).
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    g = np.random.default_rng(0)
    for arr in (bits, g.permutation(bits)):
        x = torch.from_numpy(arr.view(np.int16).copy()).view(torch.bfloat16).reshape(512, 128)
        run_both(x, True, True)


def test_weight_sync_tensor_full_size_sampled_rows():
    # Full-size Qwen3-8B gate_up weight (24576 x 4096), quantized on the GPU in the bench's launch
    # configuration; 96 sampled rows compared with the oracle (rows are independent rowwise).
    W = synth.sync_weight(0, 2, device="cuda")
    q, s_swz, _, _ = mx.quantize(W, True, False, swizzle=True)
    torch.cuda.synchronize()
    M, K = W.shape
    rows = np.sort(np.random.default_rng(1).choice(M, 96, replace=False))
    rows[0], rows[-1] = 0, M - 1
    xr = W[torch.from_numpy(rows).cuda()].cpu()
    qo, so = oracle.quantize_rowwise(xr)
    assert np.array_equal(to_np(q[torch.from_numpy(rows).cuda()]), qo)
    pos = scale_positions(M, K // 32)
    s_np = to_np(s_swz)
    assert np.array_equal(s_np[pos[rows]], so)


def test_update_step_columnwise_full_size_sampled():
    # Config "update": dY 12288 x 12288, row + col in one pass; sampled columns of dY quantized by the
    # oracle (a column of dY is a row of dY^T).
    _, _, dY = synth.update_inputs(device="cuda")
    qr, sr, qc, sc = mx.quantize(dY, True, True, swizzle=True)
    torch.cuda.synchronize()
    M, K = dY.shape
    g = np.random.default_rng(2)
    cols = np.sort(g.choice(K, 24, replace=False))
    cols[-1] = K - 1
    xc = dY[:, torch.from_numpy(cols).cuda()].t().contiguous().cpu()     # [24, M]
    qo, so = oracle.quantize_rowwise(xc)
    assert np.array_equal(to_np(qc[torch.from_numpy(cols).cuda()]), qo)
    pos = scale_positions(K, M // 32)
    assert np.array_equal(to_np(sc)[pos[cols]], so)
    rows = np.sort(g.choice(M, 24, replace=False))
    xr = dY[torch.from_numpy(rows).cuda()].cpu()
    qo, so = oracle.quantize_rowwise(xr)
    assert np.array_equal(to_np(qr[torch.from_numpy(rows).cuda()]), qo)
    pos = scale_positions(M, K // 32)
    assert np.array_equal(to_np(sr)[pos[rows]], so)


@pytest.mark.parametrize("rowwise,colwise", [(True, False), (True, True), (False, True)])
@pytest.mark.parametrize("swizzle", [True, False])
def test_quantize_multi_matches_oracle(rowwise, colwise, swizzle, quant_variant):
    # Several tensors of mixed shapes (ragged, tiny, empty, strided) in one launch.
    shapes = [(256, 512), (32, 96), (160, 288), (0, 64), (384, 1056), (96, 32), (1024, 128)]
    xs = []
    for i, (M, K) in enumerate(shapes):
        x = synth.special_bf16((M, K), seed=i) if i == 2 else synth.normal_bf16((M, K), std=2.0 ** i, seed=i,
                                                                                 outlier_frac=0.01, outlier_scale=60.0)
        xs.append(x)
    dev = [x.cuda() for x in xs]
    big = torch.zeros((384, 1096), dtype=torch.bfloat16, device="cuda")      # strided view (ld % 8 == 0)
    big[:, :1056] = dev[4]
    dev[4] = big[:, :1056]
    outs = mx.quantize_multi(dev, rowwise, colwise, swizzle)
    torch.cuda.synchronize()
    for x, (q_row, s_row, q_col, s_col) in zip(xs, outs):
        if x.shape[0] == 0:
            continue
        if rowwise:
            q, s = oracle.quantize_rowwise(x)
            assert np.array_equal(to_np(q_row), q)
            assert np.array_equal(to_np(s_row), oracle.swizzle(s) if swizzle else s)
        if colwise:
            qT, sT = oracle.quantize_colwise(x)
            assert np.array_equal(to_np(q_col), qT)
            assert np.array_equal(to_np(s_col), oracle.swizzle(sT) if swizzle else sT)


def test_quantize_multi_more_tensors_than_one_launch_holds(quant_variant):
    # 400 small tensors: split over several launches inside one call.
    xs = [synth.normal_bf16((32 * (1 + i % 5), 64 * (1 + i % 3)), seed=100 + i) for i in range(400)]
    outs = mx.quantize_multi([x.cuda() for x in xs], True, False, True)
    torch.cuda.synchronize()
    for x, (q_row, s_row, _, _) in zip(xs, outs):
        q, s = oracle.quantize_rowwise(x)
        assert np.array_equal(to_np(q_row), q) and np.array_equal(to_np(s_row), oracle.swizzle(s))


def test_empty_is_noop():
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    q, s, _, _ = mx.quantize(x, True, False, swizzle=False)
    assert q.numel() == 0
