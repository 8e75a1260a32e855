"""Self-check probe of synchronized sampler weights.

"End-to-End MXFP8 Reinforcement Learning on Blackwell" (Table 11, "self-check"; Table 10, F3 and
F4) checks at every synchronization that the sampler's kernels read what the learner's grid says.
A sampler holds derived state besides the E4M3 elements: the scale layout its GEMM reads, and for
MoE the per-expert arrangement. A stale derived copy (F3: an interleaved scale copy the sync never
rebuilt; F4: an in-place expert repack that kept shape and dtype) passes any shape check. The
probe reads the kernel's output instead of the state.

It runs the sampler's GEMM on probe activations twice -- over the sampler's derived state and over
state derived afresh from the synchronized BF16 weights -- and compares the two BF16 outputs byte
for byte on the device. The GEMM is deterministic (each output tile is computed by one CTA pair
in a fixed K order), so a healthy sampler gives exactly 0 mismatches and any mismatch means stale
or wrong derived state. Every step runs in libmx's kernels (quantize, scale layout, GEMM, byte
comparison); results stay on the device, so the probe can run inside a captured CUDA graph.
"""
from __future__ import annotations

import torch

from . import mx


def probe_dense(x: torch.Tensor, w: torch.Tensor, sampler_q: torch.Tensor, sampler_s_swz: torch.Tensor,
                out: torch.Tensor | None = None):
    """Probe one linear layer.

    x: probe activations [T, K] BF16 (CUDA); w: the synchronized BF16 weight [N, K];
    sampler_q, sampler_s_swz: the sampler's E4M3 elements [N, K] and its tensor-core scale layout.
    Returns (mismatches, first_index): 1-element int64 device tensors over the output bytes.
    """
    qx, sx, _, _ = mx.quantize(x)
    qf, sf, _, _ = mx.quantize(w)
    y_sampler = mx.gemm(qx, sx, sampler_q, sampler_s_swz)
    y_fresh = mx.gemm(qx, sx, qf, sf)
    return mx.grid_equal(y_sampler, y_fresh, out=out)


def probe_experts(x: torch.Tensor, counts, row_offsets: torch.Tensor, w: torch.Tensor, sampler_q: torch.Tensor,
                  sampler_s_swz: torch.Tensor, out: torch.Tensor | None = None):
    """Probe one MoE expert GEMM.

    x: probe tokens [sum(counts), K] BF16, grouped by expert; counts: tokens per expert (host);
    row_offsets: the same as int32 CUDA offsets [G + 1]; w: synchronized BF16 expert weights
    [G, N, K]; sampler_q [G, N, K] and sampler_s_swz: the sampler's elements and concatenated
    per-expert scale layouts. Returns (mismatches, first_index) device tensors over the output bytes.
    """
    G, N, K = w.shape
    qx, sx_raw, _, _ = mx.quantize(x, swizzle=False)
    sx = mx.swizzle_scales(sx_raw, list(counts))
    qf, sf, _, _ = mx.quantize(w.reshape(G * N, K))
    y_sampler = mx.grouped_gemm(qx, sx, sampler_q, sampler_s_swz, row_offsets)
    y_fresh = mx.grouped_gemm(qx, sx, qf.reshape(G, N, K), sf, row_offsets)
    return mx.grid_equal(y_sampler, y_fresh, out=out)
