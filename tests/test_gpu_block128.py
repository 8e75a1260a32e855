"""GPU parity: mx_quantize_block128 (FP8 blockwise, one FP32 or power-of-two scale per 128 x 128
block) against the oracle, bit for bit: codes, and scales as fp32 values (NaN where the block holds
NaN or Inf)."""
import numpy as np
import pytest
import torch

import oracle
from helpers import to_np
from mxfp8_block_scaled_07_b200 import mx, synth

pytestmark = pytest.mark.gpu


def check(x_cpu, pow2, ld_pad=0):
    M, K = x_cpu.shape
    if ld_pad:
        big = torch.zeros((M, K + ld_pad), dtype=torch.bfloat16)
        big[:, :K] = x_cpu
        xg = big.cuda()[:, :K]
    else:
        xg = x_cpu.cuda()
    q, s = mx.quantize_block128(xg, pow2)
    torch.cuda.synchronize()
    qo, so = oracle.quantize_block128(x_cpu, pow2)
    assert np.array_equal(to_np(q), qo), "codes"
    sg = s.cpu().numpy()
    assert np.array_equal(np.isnan(sg), np.isnan(so)) and np.array_equal(sg[~np.isnan(sg)], so[~np.isnan(so)]), "scales"


@pytest.mark.parametrize("shape", [(1, 32), (128, 128), (130, 160), (300, 544), (257, 4128), (1024, 96)])
@pytest.mark.parametrize("pow2", [False, True])
def test_block128_ragged_shapes(shape, pow2):
    x = synth.normal_bf16(shape, std=0.02, seed=shape[0] + shape[1], outlier_frac=1e-3, outlier_scale=50.0)
    check(x, pow2)


@pytest.mark.parametrize("pow2", [False, True])
def test_block128_special_values_and_strides(pow2):
    x = synth.special_bf16((256, 384), seed=4)
    check(x, pow2)
    z = torch.zeros((200, 256), dtype=torch.bfloat16)
    z[150:, 200:] = 1e-37                     # block (1, 1): amax / 448 is an FP32 subnormal
    z[:20, :30] = -3e-30                      # block (0, 0): tiny but normal scale
    check(z, pow2, ld_pad=64)


def test_block128_full_size_weight_sampled_slabs():
    # Qwen3-8B gate_up (24576 x 4096): the first and last 128-row slabs against the oracle (a slab's
    # blocks depend on that slab only).
    W = synth.sync_weight(0, 2, device="cuda")
    for pow2 in (False, True):
        q, s = mx.quantize_block128(W, pow2)
        torch.cuda.synchronize()
        for r0 in (0, W.shape[0] - 128):
            qo, so = oracle.quantize_block128(W[r0:r0 + 128].cpu(), pow2)
            assert np.array_equal(to_np(q[r0:r0 + 128]), qo)
            assert np.array_equal(s[r0 // 128].cpu().numpy(), so[0])
