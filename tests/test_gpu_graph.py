"""The C-ABI calls are asynchronous on the caller's stream, allocate nothing and never synchronize,
so a whole learner micro-step (quantize, GEMM, grouped GEMM, byte checks) captures into one CUDA
graph. Replaying the graph after new inputs are written in place must give exactly what the same
calls give when run eagerly on those inputs (the pages' fixed per-micro-batch cost, Table 6 and
Table 7, is what such a graph removes)."""
import numpy as np
import pytest
import torch

from helpers import to_np
from mxfp8_block_scaled_07_b200 import mx, synth

pytestmark = pytest.mark.gpu


def step(X, W, Xg, Wg, offs, counts, bufs):
    qx, qw, qxg, sxg_raw, sxg, qwg, C, Cg, ge, ref, fused_res, fused_outs = bufs
    mx.quantize(X, True, True, out=qx)
    mx.quantize(W, True, False, out=qw)
    mx.gemm(qx[0], qx[1], qw[0], qw[1], out=C)
    mx.quantize(Xg, True, False, swizzle=False, out=qxg)
    mx.swizzle_scales(qxg[1], counts, out=sxg)
    G, N, K = Wg.shape
    mx.grouped_gemm(qxg[0], sxg, qwg[0].view(G, N, K), qwg[1], offs, out=Cg)
    mx.grid_equal(qx[0], ref[0], out=ge)
    mx.quantize_compare_multi([W], [(ref[1], ref[2])], outs=fused_outs, results=fused_res)


def test_learner_step_replays_in_a_cuda_graph():
    dev = torch.device("cuda")
    M, N, K = 512, 768, 1024
    counts = [100, 0, 300, 112]
    G, Ng = len(counts), 256
    X = synth.normal_bf16((M, K), seed=1).to(dev)
    W = synth.normal_bf16((N, K), std=0.02, seed=2).to(dev)
    Xg = synth.normal_bf16((sum(counts), K), seed=3).to(dev)
    Wg = synth.normal_bf16((G, Ng, K), std=0.02, seed=4).to(dev)
    offs = torch.tensor(synth.group_offsets(counts), dtype=torch.int32, device=dev)
    qwg = mx.quantize(Wg.reshape(G * Ng, K), True, False)
    ref_x = mx.quantize(X, True, False)
    ref_w = mx.quantize(W, True, False)
    qxg = mx.quantize(Xg, True, False, swizzle=False)
    bufs = (mx.quantize(X, True, True), mx.quantize(W, True, False), qxg, qxg[1],
            mx.swizzle_scales(qxg[1], counts), qwg,
            torch.empty((M, N), dtype=torch.bfloat16, device=dev),
            torch.empty((sum(counts), Ng), dtype=torch.bfloat16, device=dev),
            torch.empty(2, dtype=torch.int64, device=dev),
            (ref_x[0], ref_w[0], ref_w[1]),
            torch.empty((2, 2), dtype=torch.int64, device=dev),
            [(torch.empty_like(ref_w[0]), torch.empty_like(ref_w[1]), None, None)])
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step(X, W, Xg, Wg, offs, counts, bufs)                 # warm-up on the capture stream's side
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(X, W, Xg, Wg, offs, counts, bufs)

    # New inputs, written in place; W changes in one row so the byte checks see differences.
    X.copy_(synth.normal_bf16((M, K), seed=11).to(dev))
    Xg.copy_(synth.normal_bf16((sum(counts), K), seed=13).to(dev))
    W[5] *= 3
    graph.replay()
    torch.cuda.synchronize()
    got = [t.clone() for t in (bufs[0][0], bufs[0][1], bufs[0][2], bufs[0][3], bufs[6], bufs[7], bufs[8],
                               bufs[10], bufs[11][0][0], bufs[11][0][1])]

    # The same calls, eagerly, into fresh buffers.
    qx = mx.quantize(X, True, True)
    qw = mx.quantize(W, True, False)
    C = mx.gemm(qx[0], qx[1], qw[0], qw[1])
    q2 = mx.quantize(Xg, True, False, swizzle=False)
    s2 = mx.swizzle_scales(q2[1], counts)
    Cg = mx.grouped_gemm(q2[0], s2, qwg[0].view(G, Ng, K), qwg[1], offs)
    ge = torch.cat(mx.grid_equal(qx[0], ref_x[0]))
    fo, fc, ff = mx.quantize_compare_multi([W], [(ref_w[0], ref_w[1])])
    torch.cuda.synchronize()
    want = [qx[0], qx[1], qx[2], qx[3], C, Cg, ge, torch.stack([fc, ff]), fo[0][0], fo[0][1]]
    for i, (a, b) in enumerate(zip(got, want)):
        assert torch.equal(a, b), i
    # The replayed checks saw the changes: X's codes differ from the old grid, W's row 5 differs.
    assert to_np(got[6])[0] > 0
    d = np.flatnonzero(to_np(got[8]).reshape(-1) != to_np(ref_w[0]).reshape(-1))
    assert to_np(got[7])[0, 0] == len(d) > 0 and to_np(got[7])[1, 0] == d[0]
