"""Seeded synthetic inputs shaped like the paper's workloads.

This module only draws random numbers; it holds none of the quantization or GEMM
arithmetic. Both the CUDA path and the CPU oracle consume what it returns, so neither side
can feed the other.

Shapes follow "End-to-End MXFP8 Reinforcement Learning on Blackwell" (arXiv 2610.34915):
Table 2 (Qwen3-8B dense; Qwen3-30B-A3B with 128 experts, top-8; dynamic micro-batches of
12 288 tokens/GPU for the dense update and 20 480 tokens/GPU for MoE) and Table 5 (the
micro-batch sweep 1.3k / 2.6k / 5.2k / 10.3k tokens). Qwen3-8B linear shapes: qkv 6144x4096,
o 4096x4096, gate_up 24576x4096, down 4096x12288 (36 layers). Qwen3-30B-A3B expert shapes:
gate_up 1536x2048, down 2048x768. Values are drawn from the distributions stated beside each
generator; no dataset or checkpoint is used.

Small tensors are drawn with a CPU ``torch.Generator``; large ones (``device="cuda"``) with a
device generator, which is deterministic for a given seed, shape and GPU model.
"""
from __future__ import annotations

import math

import torch

# Qwen3-8B per-layer linear weights [out_features, in_features] (TP=1 shapes).
QWEN3_8B_LINEARS = (("qkv", 6144, 4096), ("o", 4096, 4096), ("gate_up", 24576, 4096), ("down", 4096, 12288))
QWEN3_8B_LAYERS = 36
QWEN3_8B_HIDDEN = 4096
# Qwen3-30B-A3B MoE layer.
MOE_TOKENS = 20480
MOE_HIDDEN = 2048
MOE_EXPERTS = 128
MOE_TOPK = 8
MOE_INTER = 768          # per-expert intermediate size; gate_up has 2 * 768 = 1536 rows
MOE_ZIPF_S = 1.1
FWD_TOKENS = (1300, 5200, 10300)
UPDATE_TOKENS = 12288


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, std: float = 1.0, seed: int = 0, device="cpu", outlier_frac: float = 0.0,
                outlier_scale: float = 1.0) -> torch.Tensor:
    """N(0, std^2) in float32, a Bernoulli(outlier_frac) subset multiplied by outlier_scale,
    then rounded to BF16 (round-to-nearest-even)."""
    g = _gen(seed, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    if outlier_frac > 0.0:
        mask = torch.rand(shape, generator=g, device=device, dtype=torch.float32) < outlier_frac
        x = torch.where(mask, x * outlier_scale, x)
        del mask
    return x.to(torch.bfloat16)


def pr1_inputs(device="cpu"):
    """A[256x512], B[128x512]: N(0,1), seed 0, 1% of elements scaled x100."""
    g = _gen(0, device)
    out = []
    for shape in ((256, 512), (128, 512)):
        x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        mask = torch.rand(shape, generator=g, device=device, dtype=torch.float32) < 0.01
        out.append(torch.where(mask, x * 100.0, x).to(torch.bfloat16))
    return out[0], out[1]


def sync_weight(layer: int, idx: int, device="cpu", rows: int | None = None, cols: int | None = None):
    """Qwen3-8B BF16 master weight `idx` (0 qkv, 1 o, 2 gate_up, 3 down) of `layer`:
    N(0, 0.02^2) with 0.1% outliers x50, seed = layer * 4 + idx. `rows`/`cols` cut a smaller
    tensor with the same recipe (used by tests)."""
    _, r, c = QWEN3_8B_LINEARS[idx]
    return normal_bf16((rows or r, cols or c), std=0.02, seed=layer * 4 + idx, device=device,
                       outlier_frac=1e-3, outlier_scale=50.0)


def fwd_activations(M: int, K: int = QWEN3_8B_HIDDEN, seed: int = 1000, device="cpu"):
    """Activations [M, K]: N(0,1) times a per-channel lognormal(0,1) scale (one per column)."""
    g = _gen(seed, device)
    ch = torch.exp(torch.randn((1, K), generator=g, device=device, dtype=torch.float32))
    x = torch.randn((M, K), generator=g, device=device, dtype=torch.float32) * ch
    return x.to(torch.bfloat16)


def update_inputs(tokens: int = UPDATE_TOKENS, hidden: int = QWEN3_8B_HIDDEN, out: int = 12288,
                  device="cpu", seed: int = 2000):
    """One dense update micro-batch: X[tokens, hidden] N(0,1); W[out, hidden] N(0, 0.02^2);
    dY[tokens, out] N(0, 1e-3^2)."""
    X = normal_bf16((tokens, hidden), 1.0, seed, device)
    W = normal_bf16((out, hidden), 0.02, seed + 1, device)
    dY = normal_bf16((tokens, out), 1e-3, seed + 2, device)
    return X, W, dY


def zipf_topk_routing(tokens: int = MOE_TOKENS, experts: int = MOE_EXPERTS, topk: int = MOE_TOPK,
                      s: float = MOE_ZIPF_S, seed: int = 3000):
    """Expert loads for top-k routing with Zipf(s) popularity. Each expert gets a rank from a
    seeded permutation, p_i ~ rank_i^-s; every token draws `topk` distinct experts by Gumbel
    top-k on log p. Returns the per-expert row counts (int64 CPU tensor, sums to tokens*topk)."""
    g = _gen(seed, "cpu")
    ranks = torch.randperm(experts, generator=g) + 1
    logp = -s * torch.log(ranks.to(torch.float64))
    counts = torch.zeros(experts, dtype=torch.int64)
    chunk = 4096
    for t0 in range(0, tokens, chunk):
        n = min(chunk, tokens - t0)
        u = torch.rand((n, experts), generator=g, dtype=torch.float64).clamp_(1e-300, 1.0)
        gumbel = -torch.log(-torch.log(u))
        top = torch.topk(logp + gumbel, topk, dim=1).indices
        counts += torch.bincount(top.reshape(-1), minlength=experts)
    return counts


def group_offsets(counts) -> list[int]:
    off = [0]
    for c in counts.tolist() if hasattr(counts, "tolist") else counts:
        off.append(off[-1] + int(c))
    return off


def moe_inputs(device="cpu", counts=None, hidden: int = MOE_HIDDEN, inter: int = MOE_INTER,
               experts: int = MOE_EXPERTS, seed: int = 4000):
    """Qwen3-30B-A3B MoE layer: X_perm[sum(counts), hidden] and H[sum(counts), inter] N(0,1)
    (rows already grouped by expert); W1[E, 2*inter, hidden], W2[E, hidden, inter] N(0, 0.02^2)."""
    if counts is None:
        counts = zipf_topk_routing(experts=experts)
    rows = int(sum(int(c) for c in counts))
    Xp = normal_bf16((rows, hidden), 1.0, seed, device)
    H = normal_bf16((rows, inter), 1.0, seed + 1, device)
    W1 = normal_bf16((experts, 2 * inter, hidden), 0.02, seed + 2, device)
    W2 = normal_bf16((experts, hidden, inter), 0.02, seed + 3, device)
    return counts, Xp, H, W1, W2


def random_bytes(n: int, seed: int = 0, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    return torch.randint(0, 256, (n,), generator=g, device=device, dtype=torch.uint8)


def special_bf16(shape, seed: int = 0) -> torch.Tensor:
    """Adversarial BF16 patterns for the quantizer: random bit patterns (all exponents, signs,
    subnormals, zeros), sprinkled with +-0, +-Inf and NaN; about 1% of 32-blocks hold a NaN or
    an infinity and about 3% are entirely +-0."""
    g = _gen(seed, "cpu")
    numel = math.prod(shape)
    bits = torch.randint(0, 1 << 16, (numel,), generator=g, dtype=torch.int32)
    # Mostly finite: re-draw patterns whose exponent field is all ones.
    expo = (bits >> 7) & 0xFF
    finite = torch.randint(0, 1 << 16, (numel,), generator=g, dtype=torch.int32) & 0x7F7F
    bits = torch.where(expo == 0xFF, finite, bits)
    # Narrow the exponent spread block by block so the scale rule is exercised across the range.
    nblk = numel // 32
    center = torch.randint(1, 254, (nblk,), generator=g, dtype=torch.int32).repeat_interleave(32)
    spread = torch.randint(-12, 1, (numel,), generator=g, dtype=torch.int32)
    newexp = (center + spread).clamp(0, 254)
    mixed = (bits & 0x807F) | (newexp << 7)
    use_mixed = torch.rand(nblk, generator=g).repeat_interleave(32) < 0.8
    bits = torch.where(use_mixed, mixed, bits)
    # Specials.
    blk_kind = torch.rand(nblk, generator=g).repeat_interleave(32)
    pos = torch.randint(0, 32, (nblk,), generator=g).repeat_interleave(32)
    lane = torch.arange(numel) % 32
    spec = torch.tensor([0x7F80, 0xFF80, 0x7FC0, 0xFFC1, 0x7F81], dtype=torch.int32)
    pick = spec[torch.randint(0, len(spec), (numel,), generator=g)]
    bits = torch.where((blk_kind < 0.01) & (lane == pos), pick, bits)
    zero = torch.where(torch.rand(numel, generator=g) < 0.5, 0x0000, 0x8000).to(torch.int32)
    bits = torch.where((blk_kind > 0.97), zero, bits)
    bits = torch.where(bits >= 32768, bits - 65536, bits)
    return bits.to(torch.int16).view(torch.bfloat16).reshape(shape)
