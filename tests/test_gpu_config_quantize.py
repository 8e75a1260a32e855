"""GPU parity, bit for bit, of the activation quantizations of the forward and MoE workloads at full
size, in the launch configuration bench.py times (shapes from "End-to-End MXFP8 Reinforcement
Learning on Blackwell", Table 5: micro-batches of 1.3k / 5.2k / 10.3k tokens on the Qwen3-8B
hidden size 4096; Table 2: the Qwen3-30B-A3B MoE layer, 20 480 tokens routed top-8 over 128
experts with Zipf(1.1) loads, hidden 2048, expert intermediate 768).

Every check compares sampled rows with the oracle: the E4M3 codes, the scale bytes at their
positions in the tensor-core layout (the grouped layout for the MoE operands, each expert padded
to 128 rows), and every pad byte of the layout (0)."""
import numpy as np
import pytest
import torch

from helpers import check_sampled_rows
from mxfp8_block_scaled_07_b200 import mx, synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M", synth.FWD_TOKENS)
def test_fwd_activations_full_size(M):
    # X [M, 4096]: N(0,1) times a per-channel lognormal(0,1) scale; rowwise with the fused layout.
    X = synth.fwd_activations(M, device="cuda")
    q, s_swz, _, _ = mx.quantize(X, True, False, swizzle=True)
    torch.cuda.synchronize()
    g = np.random.default_rng(M)
    rows = np.concatenate([[0, M - 1, (M // 128) * 128, (M // 128) * 128 - 1], g.integers(0, M, 60)])
    check_sampled_rows(X, q, s_swz, rows, what=f"fwd activations {M}x4096")


@pytest.mark.parametrize("which", ["X_perm", "H"])
def test_moe_activations_full_size(which):
    # X_perm [163840, 2048] (gate_up's A operand) and H [163840, 768] (down's A operand), grouped by
    # expert: rowwise codes and raw scales, then the grouped tensor-core layout from mx_swizzle_scales.
    counts, Xp, H, _, _ = synth.moe_inputs(device="cuda")
    counts = [int(c) for c in counts]
    x = Xp if which == "X_perm" else H
    q, s_raw, _, _ = mx.quantize(x, True, False, swizzle=False)
    s_grp = mx.swizzle_scales(s_raw, counts)
    torch.cuda.synchronize()
    off = synth.group_offsets(counts)
    g = np.random.default_rng(len(which))
    rows = []
    for e, n in enumerate(counts):
        if n:
            rows += [off[e], off[e + 1] - 1, *(off[e] + g.integers(0, n, 2))]
    check_sampled_rows(x, q, s_raw, rows, swizzled=False, what=f"moe {which} raw scales")
    check_sampled_rows(x, q, s_grp, rows, group_rows=counts, what=f"moe {which} grouped layout")
