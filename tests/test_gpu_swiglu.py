"""GPU parity: mx_grouped_gemm_swiglu_quant (expert gate_up GEMM with SwiGLU and the MXFP8 rule in
its epilogue) against the oracle: grouped GEMM in fp64, SwiGLU in fp64, the rowwise MXFP8 rule.

The kernel computes h in fp32 from an fp32 accumulator, so h differs from the fp64 value by at most
the GEMM's error bound carried through SwiGLU plus a few fp32 roundings. Where that much uncertainty
straddles a rounding boundary, either neighbouring code is correct; where a block's amax lies that
close to a power of two, either scale is. The check therefore accepts, per element, exactly the
codes that some value within the bound of h rounds to under the kernel's scale, accepts per block
the scales of amax within the bound, and requires the unambiguous majority to be bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import scale_positions, to_np
from mxfp8_block_scaled_07_b200 import mx, synth

pytestmark = pytest.mark.gpu


def interleave_gate_up(w):
    """[G, 2n, K] gate rows then up rows -> rows interleaved per 128 (the fused kernel's order)."""
    G, n2, K = w.shape
    n = n2 // 2
    return w.view(G, 2, n // 128, 128, K).permute(0, 2, 1, 3, 4).reshape(G, n2, K).contiguous()


def check_against_oracle(gu, abs_sum, q_k, s_k):
    """gu, abs_sum: oracle fp64 gate_up product and sum |a b| [rows, 2n]; q_k [rows, n] codes and
    s_k [rows, n/32] scales from the kernel. Returns the fraction of bit-exact codes."""
    rows, n2 = gu.shape
    n = n2 // 2
    h_ref, q_ref, s_ref = oracle.swiglu_quantize(gu)
    g, u = gu[:, :n], gu[:, n:]
    sig = 1.0 / (1.0 + np.exp(-g))
    silu = g * sig
    # |dh| <= |dh/dg| dg + |dh/du| du + fp32 roundings: __expf (relative error about
    # (2 + 1.2 |g|) ulps), __fdividef (2 ulps) and the two products.
    tol_g, tol_u = 1e-5 * abs_sum[:, :n] + 1e-30, 1e-5 * abs_sum[:, n:] + 1e-30
    d = (np.abs(u * (sig + g * sig * (1.0 - sig))) * tol_g + np.abs(silu) * tol_u
         + (8.0 + 2.0 * np.abs(g)) * 2.0 ** -23 * np.abs(h_ref))
    hb, db = h_ref.reshape(rows, n // 32, 32), d.reshape(rows, n // 32, 32)
    amax = np.abs(hb).max(axis=2)
    dmax = db.max(axis=2)
    s_lo = np.vectorize(oracle.e8m0_scale)(np.maximum(amax - dmax, 0.0))
    s_hi = np.vectorize(oracle.e8m0_scale)(amax + dmax)
    assert np.all((s_k >= s_lo) & (s_k <= s_hi)), "scale outside what the bound allows"
    e = s_k.astype(np.int64)[:, :, None] - 127
    v = np.ldexp(hb, -e)
    dv = np.ldexp(db, -e)
    lo = oracle.e4m3_encode_array(v - dv).reshape(v.shape)
    hi = oracle.e4m3_encode_array(v + dv).reshape(v.shape)
    dec = np.array([oracle.e4m3_decode(c) for c in range(256)])
    kv = dec[q_k.reshape(v.shape)]
    assert np.all((kv >= dec[lo]) & (kv <= dec[hi])), "code outside what the bound allows"
    exact = np.mean(q_k == q_ref)
    assert np.mean(s_k == s_ref) > 0.999
    return exact


def test_fused_swiglu_quant_ragged_experts():
    counts = [40, 0, 130, 7, 256, 3, 64, 100, 129, 1]
    G, n, K = len(counts), 256, 512
    rows = sum(counts)
    off = synth.group_offsets(counts)
    X = synth.normal_bf16((rows, K), std=1.0, seed=91)
    W = synth.normal_bf16((G, 2 * n, K), std=0.02, seed=92, outlier_frac=1e-3, outlier_scale=20.0)
    # Oracle: quantize both operands, grouped GEMM in fp64 on the natural gate|up order.
    qx_o, sx_o = oracle.quantize_rowwise(X)
    qw_o, sw_o = oracle.quantize_rowwise(W.reshape(G * 2 * n, K))
    gu, abs_sum = oracle.grouped_gemm(qx_o, sx_o, qw_o.reshape(G, 2 * n, K), sw_o.reshape(G, 2 * n, K // 32), off)
    # Kernel.
    Xd = X.cuda()
    qx, sx_raw, _, _ = mx.quantize(Xd, swizzle=False)
    sx = mx.swizzle_scales(sx_raw, counts)
    Wi = interleave_gate_up(W.cuda())
    qw, sw, _, _ = mx.quantize(Wi.reshape(G * 2 * n, K))
    offd = torch.tensor(off, dtype=torch.int32, device="cuda")
    hq, hs = mx.grouped_gemm_swiglu_quant(qx, sx, qw.reshape(G, 2 * n, K), sw, offd, counts)
    assert mx.device_error() == 0
    # Scales: read back from the grouped layout (pad bytes must be 0).
    hs_np = to_np(hs)
    pos = scale_positions(rows, n // 32, counts)
    pad = np.ones(hs_np.size, bool)
    pad[pos.reshape(-1)] = False
    assert np.all(hs_np[pad] == 0), "layout pad bytes"
    exact = check_against_oracle(gu, abs_sum, to_np(hq), hs_np[pos])
    assert exact > 0.99
    print(f"fused SwiGLU+quant: {exact:.5f} of codes bit-exact")


def test_fused_swiglu_quant_full_size_moe_sampled():
    # Qwen3-30B-A3B MoE gate_up: 163840 rows, n = 768, K = 2048, 128 experts (Zipf loads); the
    # oracle recomputes the first and last row of every expert and 64 random rows.
    counts, Xp, _, W1, _ = synth.moe_inputs(device="cuda")
    counts = [int(c) for c in counts]
    G, n2, K = W1.shape
    n = n2 // 2
    off = synth.group_offsets(counts)
    qx, sx_raw, _, _ = mx.quantize(Xp, swizzle=False)
    sx = mx.swizzle_scales(sx_raw, counts)
    qw, sw, _, _ = mx.quantize(interleave_gate_up(W1).reshape(G * n2, K))
    offd = torch.tensor(off, dtype=torch.int32, device="cuda")
    hq, hs = mx.grouped_gemm_swiglu_quant(qx, sx, qw.reshape(G, n2, K), sw, offd, counts)
    assert mx.device_error() == 0
    g = np.random.default_rng(5)
    rows = sorted(set([o for o, c in zip(off[:-1], counts) if c] + [o + c - 1 for o, c in zip(off[:-1], counts) if c]
                      + list(g.integers(0, off[-1], 64))))
    expert = np.searchsorted(np.asarray(off), np.asarray(rows), side="right") - 1
    qx_o, sx_o = oracle.quantize_rowwise(Xp[torch.tensor(rows, device="cuda")].cpu())
    gu = np.empty((len(rows), n2))
    asum = np.empty((len(rows), n2))
    for e in np.unique(expert):
        sel = np.nonzero(expert == e)[0]
        qw_o, sw_o = oracle.quantize_rowwise(W1[e].cpu())
        c, a = oracle.gemm(qx_o[sel], sx_o[sel], qw_o, sw_o)
        gu[sel], asum[sel] = c, a
    pos = scale_positions(off[-1], n // 32, counts)
    hs_np = to_np(hs)
    exact = check_against_oracle(gu, asum, to_np(hq[torch.tensor(rows, device="cuda")]), hs_np[pos[rows]])
    assert exact > 0.99
    print(f"fused SwiGLU+quant (full MoE, {len(rows)} rows): {exact:.5f} of codes bit-exact")
