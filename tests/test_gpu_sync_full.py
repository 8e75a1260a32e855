"""GPU parity at the headline workload's full size, in the launch configuration bench.py times:
all 144 Qwen3-8B weights (36 layers x qkv, o, gate_up, down; 6.95 G elements) quantized rowwise
with the tensor-core scale layout by ONE mx_quantize_multi launch, then the sampler's copy
re-derived from the dequantized grid and compared by ONE mx_grid_equal_multi launch.

Checked against the oracle on sampled rows of every tensor (first, last and two random rows:
elements and the scale bytes at their positions in the layout), and through the sync invariant
of "End-to-End MXFP8 Reinforcement Learning on Blackwell" (abstract; Table 11): the sampler's
grid equals the learner's byte for byte, so every one of the 288 comparisons reports 0
mismatches and first index -1.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import scale_positions, to_np
from mxfp8_block_scaled_07_b200 import mx, synth

pytestmark = pytest.mark.gpu


def test_weight_sync_all_144_tensors_one_launch():
    shapes = [(layer, idx, r, c) for layer in range(synth.QWEN3_8B_LAYERS)
              for idx, (_, r, c) in enumerate(synth.QWEN3_8B_LINEARS)]
    assert len(shapes) == 144
    ws = [synth.sync_weight(layer, idx, device="cuda") for layer, idx, _, _ in shapes]
    outs = mx.quantize_multi(ws, True, False, True)          # one launch: 144 <= 192 tensors
    torch.cuda.synchronize()

    g = np.random.default_rng(7)
    for (layer, idx, M, K), W, (q, s_swz, _, _) in zip(shapes, ws, outs):
        rows = np.unique(np.concatenate([[0, M - 1], g.integers(0, M, 2)]))
        r_dev = torch.from_numpy(rows).cuda()
        qo, so = oracle.quantize_rowwise(W[r_dev].cpu())
        assert np.array_equal(to_np(q[r_dev]), qo), f"layer {layer} tensor {idx}: elements"
        pos = scale_positions(M, K // 32)
        assert np.array_equal(to_np(s_swz)[pos[rows]], so), f"layer {layer} tensor {idx}: scales"

    # The sampler re-derives elements and the scale layout from the dequantized BF16 grid (exact:
    # every scale here is >= 2^-124), one tensor at a time to bound memory.
    pairs = []
    samp = []
    for W, (q, s_swz, _, _) in zip(ws, outs):
        raw_q, raw_s, _, _ = mx.quantize(W, True, False, swizzle=False)
        deq = (raw_q.view(torch.float8_e4m3fn).float() *
               torch.exp2(raw_s.float() - 127.0).repeat_interleave(32, dim=1)).to(torch.bfloat16)
        del raw_q, raw_s
        qs, ss, _, _ = mx.quantize(deq, True, False, swizzle=True)
        del deq
        samp.append((qs, ss))
        pairs += [(q, qs), (s_swz, ss)]
    del ws
    cnt, first = mx.grid_equal_multi(pairs)                    # one compare launch over 288 pairs
    torch.cuda.synchronize()
    assert int(cnt.sum().item()) == 0
    assert bool((first == -1).all().item())

    # One flipped byte in the last tensor's swizzled scales is found, with its index.
    ss_last = samp[-1][1]
    ss_last[12345] ^= 1
    cnt, first = mx.grid_equal_multi(pairs)
    torch.cuda.synchronize()
    assert int(cnt.sum().item()) == 1
    assert int(cnt[-1].item()) == 1 and int(first[-1].item()) == 12345
