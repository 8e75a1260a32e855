"""GPU parity of mx_quantize_compare_multi: the weight-synchronization check ("End-to-End MXFP8
Reinforcement Learning on Blackwell", Figure 1 and Table 11's byte comparison) fused into the
quantizer. It must write exactly what mx_quantize_multi(ROWWISE | SWIZZLE) writes (checked against
the oracle) and report, for the codes and for the scale layout of every tensor, the same differing
byte count and first differing index as a byte-by-byte comparison of the written grid with the
reference (numpy, and mx_grid_equal_multi)."""
import numpy as np
import pytest
import torch

import oracle
from helpers import to_np
from mxfp8_block_scaled_07_b200 import mx, synth

pytestmark = pytest.mark.gpu

SHAPES = [(300, 96), (128, 4000), (1000, 2048), (257, 32), (0, 64), (130, 4096)]


def bf16_inputs(seed):
    xs = []
    for i, (M, K) in enumerate(SHAPES):
        xs.append(synth.normal_bf16((M, K), seed=seed + i, outlier_frac=0.01, outlier_scale=50.0).cuda())
    return xs


def numpy_compare(a, b):
    d = np.flatnonzero(to_np(a).reshape(-1) != to_np(b).reshape(-1))
    return len(d), (int(d[0]) if len(d) else -1)


def test_equal_reference_writes_the_grid_and_reports_no_difference():
    xs = bf16_inputs(11)
    ref = mx.quantize_multi(xs, True, False, True)
    refs = [(q.clone(), s.clone()) for q, s, _, _ in ref]
    outs, cnt, first = mx.quantize_compare_multi(xs, refs)
    torch.cuda.synchronize()
    assert to_np(cnt).tolist() == [0] * (2 * len(xs))
    assert to_np(first).tolist() == [-1] * (2 * len(xs))
    for x, (q, s, _, _), (qr, sr, _, _) in zip(xs, outs, ref):
        assert torch.equal(q, qr) and torch.equal(s, sr)
        if x.shape[0] == 0:
            continue
        qo, so = oracle.quantize_rowwise(x.cpu())
        assert np.array_equal(to_np(q), qo)
        assert np.array_equal(to_np(s), oracle.swizzle(so))


def test_planted_differences_are_counted_like_a_byte_comparison():
    xs = bf16_inputs(21)
    ref = mx.quantize_multi(xs, True, False, True)
    refs = [(q.clone(), s.clone()) for q, s, _, _ in ref]
    g = np.random.default_rng(5)
    # Codes: first byte of tensor 0, last byte of tensor 1, a whole 32-byte block and scattered
    # bytes of tensor 2; scales: a pad byte of tensor 3's layout (beyond its 257 rows), the first
    # byte of tensor 5's, random bytes of tensor 2's.
    refs[0][0].view(-1)[0] ^= 1
    refs[1][0].view(-1)[-1] ^= 0x80
    refs[2][0][7, 64:96] ^= 0xFF
    for i in g.integers(0, refs[2][0].numel(), 50):
        refs[2][0].view(-1)[int(i)] ^= 0x10
    refs[3][1].view(-1)[2 * 512 + 12 * 16 + 4] ^= 2     # row 300 of 257: a pad byte of the layout
    refs[5][1].view(-1)[0] ^= 4
    for i in g.integers(0, refs[2][1].numel(), 9):
        refs[2][1].view(-1)[int(i)] += 1
    outs, cnt, first = mx.quantize_compare_multi(xs, refs)
    pairs = []
    for (q, s, _, _), (qr, sr) in zip(outs, refs):
        pairs += [(q, qr), (s, sr)]
    gc, gf = mx.grid_equal_multi(pairs)
    torch.cuda.synchronize()
    expect = [numpy_compare(a, b) for a, b in pairs]
    assert to_np(cnt).tolist() == [c for c, _ in expect]
    assert to_np(first).tolist() == [f for _, f in expect]
    assert to_np(cnt).tolist() == to_np(gc).tolist() and to_np(first).tolist() == to_np(gf).tolist()
    assert to_np(cnt)[4] >= 32                               # the whole flipped block counts
    assert to_np(cnt)[7] == 1 and to_np(first)[7] == 2 * 512 + 12 * 16 + 4


def test_weight_sync_all_144_tensors_fused():
    """The headline workload: one fused launch over all 144 Qwen3-8B weights against the sampler's
    re-derived copy gives 0 differences everywhere and the same grid as the two-launch step; one
    flipped byte in the copy is found with its index."""
    ws = [synth.sync_weight(layer, idx, device="cuda") for layer in range(synth.QWEN3_8B_LAYERS)
          for idx in range(len(synth.QWEN3_8B_LINEARS))]
    learner = mx.quantize_multi(ws, True, False, True)
    samp = []
    for W in ws:
        raw_q, raw_s, _, _ = mx.quantize(W, True, False, swizzle=False)
        deq = (raw_q.view(torch.float8_e4m3fn).float() *
               torch.exp2(raw_s.float() - 127.0).repeat_interleave(32, dim=1)).to(torch.bfloat16)
        del raw_q, raw_s
        qs, ss, _, _ = mx.quantize(deq, True, False, swizzle=True)
        del deq
        samp.append((qs, ss))
    outs, cnt, first = mx.quantize_compare_multi(ws, samp)
    torch.cuda.synchronize()
    assert int(cnt.sum().item()) == 0 and bool((first == -1).all().item())
    for (q, s, _, _), (ql, sl, _, _) in zip(outs, learner):
        assert torch.equal(q, ql) and torch.equal(s, sl)
    samp[77][0].view(-1)[123457] ^= 0x40
    outs, cnt, first = mx.quantize_compare_multi(ws, samp, outs=outs)
    torch.cuda.synchronize()
    c, f = to_np(cnt), to_np(first)
    assert c.sum() == 1 and c[2 * 77] == 1 and f[2 * 77] == 123457
    assert (np.delete(f, 2 * 77) == -1).all()


def test_more_tensors_than_one_launch_holds():
    """200 tensors take two launches (192 + 8): every tensor's results land in its own slots."""
    g = np.random.default_rng(9)
    shapes = [(int(g.integers(1, 300)), 32 * int(g.integers(1, 12))) for _ in range(200)]
    xs = [synth.normal_bf16(sh, seed=100 + i).cuda() for i, sh in enumerate(shapes)]
    ref = mx.quantize_multi(xs, True, False, True)
    refs = [(q.clone(), s.clone()) for q, s, _, _ in ref]
    planted = {3: 0, 191: 5, 192: 0, 199: 7}
    for i, pos in planted.items():
        refs[i][0].view(-1)[pos] ^= 1
    outs, cnt, first = mx.quantize_compare_multi(xs, refs)
    torch.cuda.synchronize()
    c, f = to_np(cnt), to_np(first)
    for i in range(200):
        want = (1, planted[i]) if i in planted else (0, -1)
        assert (c[2 * i], f[2 * i]) == want, i
        assert c[2 * i + 1] == 0 and f[2 * i + 1] == -1, i
    for (q, s, _, _), (qr, sr, _, _) in zip(outs, ref):
        assert torch.equal(q, qr) and torch.equal(s, sr)
