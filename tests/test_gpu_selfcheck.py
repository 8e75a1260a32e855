"""GPU: the self-check probe (mxfp8_block_scaled_07_b200.selfcheck) on healthy and stale samplers.

Faults follow "End-to-End MXFP8 Reinforcement Learning on Blackwell", Table 10: F3 (the sampler's
swizzled scale copy is left from the previous weights while its elements are fresh) and F4 (an
in-place repack of the experts that keeps shape and dtype). A healthy sampler gives exactly 0
mismatching output bytes; both faults give many.

Beside the byte comparison, the probe's relative error ||y - ref|| / ||ref|| is measured against two
references computed by the CPU oracle from the same synchronized weights (the pages' MoE probe:
0.05 healthy, 1.74 with F4):
  - the oracle's MXFP8 GEMM of the learner's grid (fp64 over the oracle's own quantization of the
    BF16 activations and weights): a healthy sampler differs from it only by the BF16 rounding of
    the output and the GEMM tolerance, so <= 2^-8; a stale sampler by far more;
  - the exact fp64 product of the BF16 activations and weights (a numpy matmul): a healthy sampler
    is off by the MXFP8 quantization error (about 0.05, the pages' healthy figure).
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import to_np
from mxfp8_block_scaled_07_b200 import mx, selfcheck, synth

pytestmark = pytest.mark.gpu


def sampler_copy(w):
    """What a healthy sampler holds after a sync: the learner's grid, re-derived on the sampler
    from the dequantized BF16 weights (exact here: every scale is >= 2^-124)."""
    q0, s0, _, _ = mx.quantize(w, swizzle=False)
    deq = (q0.view(torch.float8_e4m3fn).float() * torch.exp2(s0.float() - 127.0).repeat_interleave(32, dim=1))
    q, s, _, _ = mx.quantize(deq.to(torch.bfloat16))
    return q, s


def rel_err(y, ref):
    return float(((y.float() - ref).norm() / ref.norm()).item())


def rel_err_np(y, ref):
    y = np.asarray(y, np.float64)
    return float(np.linalg.norm(y - ref) / np.linalg.norm(ref))


def bf16_f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def test_dense_probe_healthy_and_stale_scales():
    T, N, K = 256, 1024, 4096
    x = synth.fwd_activations(T, K, device="cuda")
    w_old = synth.normal_bf16((N, K), std=0.02, seed=71, device="cuda", outlier_frac=1e-3, outlier_scale=50.0)
    w = (w_old.float() + synth.normal_bf16((N, K), std=0.02, seed=72, device="cuda").float()).to(torch.bfloat16)
    ref = x.float() @ w.float().t()

    q, s = sampler_copy(w)
    cnt, first = selfcheck.probe_dense(x, w, q, s)
    torch.cuda.synchronize()
    assert int(cnt.item()) == 0 and int(first.item()) == -1
    qx, sx, _, _ = mx.quantize(x)
    healthy = rel_err(mx.gemm(qx, sx, q, s), ref)
    assert healthy < 0.1

    # F3: fresh elements, scale layout left from the previous weights.
    _, s_old = sampler_copy(w_old)
    assert not torch.equal(s_old, s)
    cnt, first = selfcheck.probe_dense(x, w, q, s_old)
    torch.cuda.synchronize()
    assert int(cnt.item()) > 0 and int(first.item()) >= 0
    y_stale = mx.gemm(qx, sx, q, s_old)
    stale = rel_err(y_stale, ref)
    assert stale > 2 * healthy

    # Against the oracle on sampled output rows: its MXFP8 GEMM of the learner's grid, and the
    # exact product of the BF16 values.
    rows = np.unique(np.concatenate([[0, T - 1], np.random.default_rng(5).integers(0, T, 22)]))
    r_dev = torch.from_numpy(rows).cuda()
    qx_o, sx_o = oracle.quantize_rowwise(x[r_dev].cpu())
    qw_o, sw_o = oracle.quantize_rowwise(w.cpu())
    ref_mx, _ = oracle.gemm(qx_o, sx_o, qw_o, sw_o)
    exact = bf16_f64(x[r_dev]) @ bf16_f64(w).T
    y_ok = to_np(mx.gemm(qx, sx, q, s)[r_dev].float())
    y_bad = to_np(y_stale[r_dev].float())
    e_ok, e_bad = rel_err_np(y_ok, ref_mx), rel_err_np(y_bad, ref_mx)
    x_ok, x_bad = rel_err_np(y_ok, exact), rel_err_np(y_bad, exact)
    assert e_ok <= 2.0 ** -8 and e_bad > 0.1
    assert x_ok < 0.1 and x_bad > 2 * x_ok
    print(f"dense probe: relative error healthy {healthy:.4f}, stale scales {stale:.4f} (torch BF16 product); "
          f"vs oracle MXFP8 GEMM: healthy {e_ok:.2e}, stale {e_bad:.4f}; vs exact product: healthy {x_ok:.4f}, "
          f"stale {x_bad:.4f}")


def test_expert_probe_healthy_and_repacked_experts():
    counts = [40, 0, 130, 7, 256, 3, 64, 100]
    G, N, K = len(counts), 256, 512
    rows = sum(counts)
    off = torch.tensor(synth.group_offsets(counts), dtype=torch.int32, device="cuda")
    x = synth.normal_bf16((rows, K), std=1.0, seed=81, device="cuda")
    w = synth.normal_bf16((G, N, K), std=0.02, seed=82, device="cuda")

    q2, s = sampler_copy(w.reshape(G * N, K))
    q = q2.reshape(G, N, K)
    cnt, first = selfcheck.probe_experts(x, counts, off, w, q, s)
    torch.cuda.synchronize()
    assert int(cnt.item()) == 0 and int(first.item()) == -1

    # F4: the experts' elements and scale layouts repacked in a different order (same shape, dtype).
    perm = [1, 0, 3, 2, 5, 4, 7, 6]
    blk = s.numel() // G                   # N = 256: each expert's scale layout is the same size
    q_bad = q[perm].contiguous()
    s_bad = s.reshape(G, blk)[perm].reshape(-1).contiguous()
    cnt, first = selfcheck.probe_experts(x, counts, off, w, q_bad, s_bad)
    torch.cuda.synchronize()
    assert int(cnt.item()) > 0 and int(first.item()) >= 0

    # Relative error against the BF16 product of each expert's synchronized weights.
    ref = torch.empty((rows, N), dtype=torch.float32, device="cuda")
    o = synth.group_offsets(counts)
    for g in range(G):
        ref[o[g]:o[g + 1]] = x[o[g]:o[g + 1]].float() @ w[g].float().t()
    qx, sx_raw, _, _ = mx.quantize(x, swizzle=False)
    sx = mx.swizzle_scales(sx_raw, counts)
    healthy = rel_err(mx.grouped_gemm(qx, sx, q, s, off), ref)
    repacked = rel_err(mx.grouped_gemm(qx, sx, q_bad, s_bad, off), ref)
    assert healthy < 0.1 and repacked > 1.0

    # Against the oracle: its grouped MXFP8 GEMM of the learner's grid, and the exact product.
    qx_o, sx_o = oracle.quantize_rowwise(x.cpu())
    qw_o, sw_o = oracle.quantize_rowwise(w.reshape(G * N, K).cpu())
    ref_mx, _ = oracle.grouped_gemm(qx_o, sx_o, qw_o.reshape(G, N, K), sw_o.reshape(G, N, K // 32), o)
    xs, ws = bf16_f64(x), bf16_f64(w)
    exact = np.concatenate([xs[o[g]:o[g + 1]] @ ws[g].T for g in range(G)])
    y_ok = to_np(mx.grouped_gemm(qx, sx, q, s, off).float())
    y_bad = to_np(mx.grouped_gemm(qx, sx, q_bad, s_bad, off).float())
    e_ok, e_bad = rel_err_np(y_ok, ref_mx), rel_err_np(y_bad, ref_mx)
    x_ok, x_bad = rel_err_np(y_ok, exact), rel_err_np(y_bad, exact)
    assert e_ok <= 2.0 ** -8 and e_bad > 1.0
    assert x_ok < 0.1 and x_bad > 1.0
    print(f"expert probe: relative error healthy {healthy:.4f}, repacked experts {repacked:.4f} (torch BF16 "
          f"product); vs oracle MXFP8 GEMM: healthy {e_ok:.2e}, repacked {e_bad:.4f}; vs exact product: "
          f"healthy {x_ok:.4f}, repacked {x_bad:.4f}")
