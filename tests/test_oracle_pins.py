"""Pins for the CPU oracle: checks against things other than the oracle itself.

- E4M3 decode and encode against torch's float8_e4m3fn conversion (a library routine) for every
  BF16 bit pattern at a sweep of block scales, and against a brute-force nearest-code search in
  exact rational arithmetic;
- hand-worked blocks of the scale rule (tests/golden/scale_rule_blocks.txt);
- the per-element error bound of the rule and the sync invariant of the paper ("End-to-End MXFP8
  Reinforcement Learning on Blackwell", abstract and Table 11: synchronized weights equal the
  learner's quantized forward operand byte for byte), i.e. quantize(dequantize(q, s)) == (q, s);
- the scale layout at hand-computed positions, as a bijection, and against the reshape/permute
  statement of the same layout (128x4 blocks of 32x16 bytes);
- the GEMM against exact integer arithmetic and against numpy's fp64 matmul;
- the byte comparison against numpy.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from mxfp8_block_scaled_07_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_bits(values) -> np.ndarray:
    t = torch.tensor(values, dtype=torch.float64)
    b = t.to(torch.bfloat16)
    finite = torch.isfinite(t)
    assert torch.equal(b.to(torch.float64)[finite], t[finite]), "fixture value not exact in BF16"
    out = b.view(torch.int16).numpy().view(np.uint16).copy()
    out[torch.isnan(t).numpy()] = 0x7FC0     # "nan" in a fixture is the positive quiet NaN
    return out


def all_finite_bf16() -> np.ndarray:
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    expo = (bits >> 7) & 0xFF
    return bits[expo != 0xFF]


def bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ---- E4M3 element format ---------------------------------------------------------------


def test_decode_matches_torch_for_all_codes():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = np.array([oracle.e4m3_decode(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(ours))
    assert nan.sum() == 2  # 0x7f and 0xff
    assert np.array_equal(ref[~nan], ours[~nan])
    assert np.array_equal(np.signbit(ref[~nan]), np.signbit(ours[~nan]))


@pytest.mark.parametrize("e", [-127, -126, -124, -120, -100, -60, -20, -9, -8, -7, -1, 0, 1, 8, 40, 100, 119])
def test_encode_every_bf16_at_scale_matches_torch(e):
    x = bits_to_f64(all_finite_bf16())
    v = np.ldexp(x, -e)                        # exact in fp64
    ours = oracle.e4m3_encode_array(v)
    # torch maps |v| >= 464 to NaN, so clamp to the saturation value first (then fp32 is exact
    # for every |v| in [2^-149, 448]; smaller magnitudes round to a signed zero either way).
    ref = torch.from_numpy(v).clamp(-448.0, 448.0).to(torch.float32).to(torch.float8_e4m3fn)
    ref = ref.view(torch.uint8).numpy()
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, f"first mismatch v={v[bad[0]]!r}: ours {ours[bad[0]]:#x} torch {ref[bad[0]]:#x}"


def _nearest_code_bruteforce(v: Fraction, negative: bool) -> int:
    """Nearest finite E4M3 value by exhaustive search; ties go to the even code; saturating."""
    table = []
    for code in range(0x7F):  # non-negative finite codes 0x00..0x7e
        expo, mant = code >> 3, code & 7
        val = Fraction(mant, 512) if expo == 0 else Fraction(8 + mant, 8) * Fraction(2) ** (expo - 7)
        table.append((val, code))
    a = abs(v)
    if a >= 448:
        code = 0x7E
    else:
        best = min(table, key=lambda t: (abs(t[0] - a), t[1] & 1))
        code = best[1]
    return code | (0x80 if negative else 0)


def test_encode_against_bruteforce_nearest():
    g = np.random.default_rng(7)
    x = bits_to_f64(all_finite_bf16())
    picks = g.choice(x.size, 2500, replace=False)
    es = g.integers(-127, 120, picks.size)
    vals = np.ldexp(x[picks], -es)
    edge = np.array([0.0, -0.0, 2.0**-10, -(2.0**-10), 3 * 2.0**-11, 3 * 2.0**-10, 5 * 2.0**-10, 448.0, 456.0,
                     464.0, 500.0, -1e30, 1.0625, 1.1875, 15.5 * 2.0**-6, 2.0**-6 * 1.0625, 240.0, 232.0])
    vals = np.concatenate([vals, edge])
    ours = oracle.e4m3_encode_array(vals)
    for v, o in zip(vals, ours):
        ref = _nearest_code_bruteforce(Fraction(float(v)), bool(np.signbit(v)))
        assert o == ref, (v, hex(o), hex(ref))


# ---- scale rule: hand-worked blocks -------------------------------------------------------


def _golden_blocks():
    out = []
    with open(os.path.join(GOLDEN, "scale_rule_blocks.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = [p.strip() for p in line.split("|")]
            name, elems, scale, codes = parts[:4]
            fill = 0.0
            for extra in parts[4:]:
                if extra.startswith("fill="):
                    fill = float(extra[5:])
            vals = [float(v) for v in elems.split()]
            out.append((name, vals, int(scale), [int(c, 16) for c in codes.split()], fill))
    return out


@pytest.mark.parametrize("case", _golden_blocks(), ids=lambda c: c[0])
def test_scale_rule_hand_worked(case):
    name, vals, scale, codes, fill = case
    block = [fill] * 32
    block[: len(vals)] = vals
    bits = bf16_bits(block).reshape(1, 32)
    q, s = oracle.quantize_rowwise(bits)
    assert s[0, 0] == scale
    assert list(q[0, : len(codes)]) == codes
    # The same block as the 2nd block of a row and as a column gives the same bytes.
    row2 = np.concatenate([bf16_bits([1.0] * 32).reshape(1, 32), bits], axis=1)
    q2, s2 = oracle.quantize_rowwise(row2)
    assert s2[0, 1] == scale and list(q2[0, 32: 32 + len(codes)]) == codes
    qT, sT = oracle.quantize_colwise(bits.reshape(32, 1))
    assert sT[0, 0] == scale and list(qT[0, : len(codes)]) == codes


def test_scale_exponent_is_floor_log2_minus_8_over_the_bf16_range():
    # Every positive normal BF16 magnitude that is a block's amax: e = floor(log2) - 8, clamped.
    for expo in range(1, 255):
        for mant in (0, 1, 64, 127):
            amax = math.ldexp(1.0 + mant / 128.0, expo - 127)
            e = max(expo - 127 - 8, -127)
            assert oracle.e8m0_scale(amax) == e + 127


# ---- error bound and the sync invariant --------------------------------------------------


def _dequant_ok_blocks(shape, seed):
    x = synth.normal_bf16(shape, std=1.0, seed=seed, outlier_frac=0.01, outlier_scale=100.0)
    return oracle._bits(x), x.to(torch.float64).numpy()


def test_elementwise_error_bound():
    bits, x = _dequant_ok_blocks((64, 256), 11)
    q, s = oracle.quantize_rowwise(bits)
    dq = oracle.dequantize(q, s)
    e = np.repeat(s.astype(np.int64) - 127, 32, axis=1)
    y = np.abs(np.ldexp(x, -e))                        # |x| in units of the block scale
    sat = y > 448
    # half an E4M3 ulp at y: 2^(max(floor(log2 y), -6) - 4)
    with np.errstate(divide="ignore"):
        ex = np.floor(np.log2(np.where(y > 0, y, 1.0)))
    half_ulp = np.ldexp(1.0, (np.maximum(ex, -6) - 4).astype(np.int64))
    err = np.abs(np.ldexp(x - dq, -e))
    assert np.all(err[~sat] <= half_ulp[~sat])
    assert np.all(err[sat] < 64)
    assert np.all(np.abs(dq) <= np.abs(x) + np.ldexp(half_ulp, e))


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_requantizing_dequantized_grid_reproduces_bytes(seed):
    # The paper's sync invariant: the sampler's copy, re-derived from the learner's grid, equals
    # the learner's bytes. Dequantized values are exact in BF16 whenever every block scale is
    # >= 2^-124 (true for these inputs), so the BF16 round trip is lossless.
    bits, _ = _dequant_ok_blocks((96, 320), seed)
    q, s = oracle.quantize_rowwise(bits)
    assert s.min() >= 3
    dq = oracle.dequantize(q, s)
    dq_bf16 = torch.from_numpy(dq).to(torch.bfloat16)
    assert np.array_equal(dq_bf16.to(torch.float64).numpy(), dq)
    q2, s2 = oracle.quantize_rowwise(dq_bf16)
    assert np.array_equal(q, q2) and np.array_equal(s, s2)
    # Columnwise too.
    qT, sT = oracle.quantize_colwise(bits)
    dqT = oracle.dequantize(qT, sT)                 # [K, M], on the columnwise grid
    qT2, sT2 = oracle.quantize_rowwise(torch.from_numpy(dqT).to(torch.bfloat16))
    assert np.array_equal(qT, qT2) and np.array_equal(sT, sT2)


def test_special_inputs_follow_policy():
    x = synth.special_bf16((64, 512), seed=5)
    bits = oracle._bits(x)
    q, s = oracle.quantize_rowwise(bits)
    f = bits_to_f64(bits.reshape(-1)).reshape(bits.shape)
    blocks = f.reshape(64, 16, 32)
    special = ~np.isfinite(blocks).all(axis=2)
    assert special.any() and (~special).any()
    assert np.all(s[special] == 0xFF)
    qb = q.reshape(64, 16, 32)
    signs = np.signbit(blocks)
    assert np.all(qb[special] == np.where(signs[special], 0xFF, 0x7F))
    zero = (blocks == 0).all(axis=2)
    assert zero.any() and np.all(s[zero] == 0)


# ---- columnwise ---------------------------------------------------------------------------


def test_colwise_is_rowwise_of_transpose_and_blocks_run_along_m():
    x = synth.normal_bf16((96, 64), seed=3)
    bits = oracle._bits(x)
    qT, sT = oracle.quantize_colwise(bits)
    assert qT.shape == (64, 96) and sT.shape == (64, 3)
    q2, s2 = oracle.quantize_rowwise(np.ascontiguousarray(bits.T))
    assert np.array_equal(qT, q2) and np.array_equal(sT, s2)
    # A single large entry at (m=40, k=5) only changes the scale of column 5's second M-block.
    big = bits.copy()
    big[40, 5] = bf16_bits([1048576.0])[0]
    qb, sb = oracle.quantize_colwise(big)
    diff = np.argwhere(sb != sT)
    assert diff.tolist() == [[5, 1]]


# ---- scale layout -------------------------------------------------------------------------


def test_swizzle_positions_hand_computed():
    # Documented sm_100 layout: block (r/128, c/4) of 512 bytes; inside, (r%32)*16 + (r%128/32)*4 + c%4.
    rows, cols = 256, 8          # 2 x 2 blocks
    s = np.zeros((rows, cols), np.uint8)
    marks = {(0, 0): 1, (1, 0): 2, (31, 0): 3, (32, 0): 4, (96, 3): 5, (0, 1): 6, (0, 4): 7, (128, 0): 8,
             (255, 7): 9, (33, 6): 10}
    for (r, c), v in marks.items():
        s[r, c] = v
    out = oracle.swizzle(s)
    assert out.size == 256 * 8
    expect = {0: 1, 16: 2, 496: 3, 4: 4, 15: 5, 1: 6, 512: 7, 1024: 8, 1024 + 512 + 511: 9, 512 + 16 + 4 + 2: 10}
    got = {int(i): int(out[i]) for i in np.nonzero(out)[0]}
    assert got == expect


def test_swizzle_padding_and_bijection():
    rows, cols = 300, 13      # pads to 384 x 16
    s = (np.arange(rows * cols) % 251 + 1).astype(np.uint8).reshape(rows, cols)
    out = oracle.swizzle(s)
    assert out.size == 384 * 16 == oracle.swizzled_size(rows, cols)
    # Track where each scale goes with a unique 16-bit tag split over two byte planes.
    tag = np.arange(rows * cols, dtype=np.int64).reshape(rows, cols)
    lo = oracle.swizzle((tag & 0xFF).astype(np.uint8)).astype(np.int64)
    hi = oracle.swizzle((tag >> 8).astype(np.uint8)).astype(np.int64)
    pos = lo | (hi << 8)
    filled = oracle.swizzle(np.ones((rows, cols), np.uint8)).astype(bool)
    assert filled.sum() == rows * cols                     # every scale lands once
    assert np.array_equal(np.sort(pos[filled]), np.arange(rows * cols))
    assert np.all(out[~filled] == 0)                       # pads are zero


def test_swizzle_matches_block_reshape_statement():
    # The same layout stated with reshapes: pad to [R', C'], view as (R'/128, 128, C'/4, 4),
    # order blocks row-block major, and store each 128x4 block as 32 rows of 4x4 bytes.
    g = np.random.default_rng(3)
    for rows, cols in [(128, 4), (256, 16), (200, 10), (1, 1), (513, 7)]:
        s = g.integers(0, 256, (rows, cols), dtype=np.uint8)
        R, C = -(-rows // 128) * 128, -(-cols // 4) * 4
        p = np.zeros((R, C), np.uint8)
        p[:rows, :cols] = s
        blocks = p.reshape(R // 128, 128, C // 4, 4).transpose(0, 2, 1, 3)     # (rb, cb, 128, 4)
        inner = blocks.reshape(-1, 4, 32, 4).transpose(0, 2, 1, 3)            # (blk, r%32, r/32, c)
        assert np.array_equal(oracle.swizzle(s), inner.reshape(-1))


def test_grouped_swizzle_is_concatenation_of_per_group_layouts():
    g = np.random.default_rng(4)
    groups = [0, 5, 128, 129, 300, 0, 1]
    cols = 24
    s = g.integers(0, 256, (sum(groups), cols), dtype=np.uint8)
    out = oracle.swizzle(s, groups)
    parts, r0 = [], 0
    for n in groups:
        if n:
            parts.append(oracle.swizzle(s[r0: r0 + n]))
        r0 += n
    assert np.array_equal(out, np.concatenate(parts))


# ---- GEMM ---------------------------------------------------------------------------------


def _int_codes(g, shape):
    """E4M3 codes of small integers -8..8 (values exact), as uint8."""
    vals = g.integers(-8, 9, shape)
    codes = oracle.e4m3_encode_array(vals.astype(np.float64)).reshape(shape)
    assert np.array_equal(np.array([oracle.e4m3_decode(c) for c in codes.reshape(-1)]).reshape(shape), vals)
    return vals, codes


def test_gemm_exact_integer_case_and_transposes():
    g = np.random.default_rng(5)
    M, N, K = 5, 7, 96
    a_int, qa = _int_codes(g, (M, K))
    b_int, qb = _int_codes(g, (N, K))
    sa = np.full((M, K // 32), 127, np.uint8)
    sb = np.full((N, K // 32), 127, np.uint8)
    c, a = oracle.gemm(qa, sa, qb, sb)
    assert np.array_equal(c, (a_int @ b_int.T).astype(np.float64))
    assert np.array_equal(a, (np.abs(a_int) @ np.abs(b_int).T).astype(np.float64))
    # Per-block scales 2^(s-127): exact values, so numpy's fp64 matmul of the dequantized operands
    # is exact too; a scale applied to the wrong K-block or operand breaks equality.
    sa = g.integers(120, 135, (M, K // 32)).astype(np.uint8)
    sb = g.integers(120, 135, (N, K // 32)).astype(np.uint8)
    c, _ = oracle.gemm(qa, sa, qb, sb)
    da = a_int * np.ldexp(1.0, np.repeat(sa.astype(np.int64) - 127, 32, axis=1))
    db = b_int * np.ldexp(1.0, np.repeat(sb.astype(np.int64) - 127, 32, axis=1))
    assert np.array_equal(c, da @ db.T)


def test_gemm_random_matches_numpy_fp64():
    A = synth.normal_bf16((48, 160), seed=8, outlier_frac=0.01, outlier_scale=100.0)
    B = synth.normal_bf16((40, 160), seed=9)
    qa, sa = oracle.quantize_rowwise(A)
    qb, sb = oracle.quantize_rowwise(B)
    c, a = oracle.gemm(qa, sa, qb, sb)
    da, db = oracle.dequantize(qa, sa), oracle.dequantize(qb, sb)
    ref = da @ db.T
    assert np.all(np.abs(c - ref) <= 1e-12 * (np.abs(da) @ np.abs(db).T))
    assert np.allclose(a, np.abs(da) @ np.abs(db).T, rtol=1e-13, atol=0)
    # and the quantized GEMM approximates the BF16 product within the rule's error.
    exact = A.to(torch.float64).numpy() @ B.to(torch.float64).numpy().T
    assert np.all(np.abs(c - exact) <= 2 ** -3 * (np.abs(A.double().numpy()) @ np.abs(B.double().numpy()).T))


def test_grouped_gemm_equals_per_group_dense():
    g = np.random.default_rng(6)
    counts = [3, 0, 17, 1, 9]
    off = np.concatenate([[0], np.cumsum(counts)])
    K, N = 64, 24
    qa = g.integers(0, 0x7E, (off[-1], K), dtype=np.uint8)
    sa = g.integers(110, 140, (off[-1], K // 32), dtype=np.uint8)
    qb = g.integers(0, 0x7E, (len(counts), N, K), dtype=np.uint8) | (g.integers(0, 2, (len(counts), N, K)) * 0x80).astype(np.uint8)
    sb = g.integers(110, 140, (len(counts), N, K // 32), dtype=np.uint8)
    c, a = oracle.grouped_gemm(qa, sa, qb, sb, off)
    for e in range(len(counts)):
        r0, r1 = off[e], off[e + 1]
        if r1 > r0:
            ce, ae = oracle.gemm(qa[r0:r1], sa[r0:r1], qb[e], sb[e])
            assert np.array_equal(c[r0:r1], ce) and np.array_equal(a[r0:r1], ae)


# ---- byte comparison ----------------------------------------------------------------------


def test_grid_equal_matches_numpy():
    g = np.random.default_rng(8)
    a = g.integers(0, 256, 10007, dtype=np.uint8)
    assert oracle.grid_equal(a, a.copy()) == (0, -1)
    b = a.copy()
    idx = np.sort(g.choice(a.size, 37, replace=False))
    b[idx] ^= g.integers(1, 256, idx.size, dtype=np.uint8)
    assert oracle.grid_equal(a, b) == (37, int(idx[0]))
    assert oracle.grid_equal(a[:0], b[:0]) == (0, -1)


# ---- SwiGLU + MXFP8 rule on the expert activation -----------------------------------------


def test_swiglu_quantize_reduces_to_the_bf16_quantizer_for_saturated_gates():
    # For gate = 2^k with k >= 6, sigmoid(gate) rounds to exactly 1 in fp64, so h = gate * up is
    # exact and BF16-representable (up BF16, gate a power of two): the result must equal the
    # (independently pinned) BF16 rowwise quantizer applied to that BF16 tensor.
    g = np.random.default_rng(21)
    rows, n = 6, 96
    up = synth.normal_bf16((rows, n), std=3.0, seed=22, outlier_frac=0.05, outlier_scale=40.0)
    gate = np.ldexp(1.0, g.integers(6, 40, (rows, n)))
    gu = np.concatenate([gate, up.double().numpy()], axis=1)
    h, q, s = oracle.swiglu_quantize(gu)
    hb = torch.from_numpy(gate * up.double().numpy()).to(torch.bfloat16)
    assert np.array_equal(hb.double().numpy(), h)          # h is exactly gate * up
    q_ref, s_ref = oracle.quantize_rowwise(hb)
    assert np.array_equal(q, q_ref) and np.array_equal(s, s_ref)


def test_swiglu_quantize_special_cases():
    n = 32
    # up = 0: h = +-0 (sign of silu(gate)); all-zero block -> scale 0, codes 0x00 / 0x80.
    gate = np.linspace(-5.0, 5.0, n)
    gu = np.concatenate([gate, np.zeros(n)])[None, :]
    h, q, s = oracle.swiglu_quantize(gu)
    assert np.all(h == 0.0) and s[0, 0] == 0
    assert np.array_equal(q[0], np.where(gate < 0, 0x80, 0x00).astype(np.uint8))
    # gate = ln 3: sigmoid = 3/4, so h = 0.75 ln(3) up.
    up = np.linspace(-2.0, 2.0, n)
    gu = np.concatenate([np.full(n, math.log(3.0)), up])[None, :]
    h, _, _ = oracle.swiglu_quantize(gu)
    assert np.allclose(h[0], 0.75 * math.log(3.0) * up, rtol=4e-16, atol=0.0)
    with pytest.raises(ValueError):
        oracle.swiglu_quantize(np.zeros((1, 2 * 48)))


def test_swiglu_odd_part_is_gate_times_up():
    # silu(x) - silu(-x) = x, so h(g, u) - h(-g, u) = g u: a check of the sign and of which half
    # is the gate.
    g = np.random.default_rng(23)
    gate = g.normal(0.0, 3.0, (4, 64))
    up = g.normal(0.0, 1.0, (4, 64))
    h1, _, _ = oracle.swiglu_quantize(np.concatenate([gate, up], axis=1))
    h2, _, _ = oracle.swiglu_quantize(np.concatenate([-gate, up], axis=1))
    assert np.allclose(h1 - h2, gate * up, rtol=1e-13, atol=1e-14)


# ---- FP8 blockwise, 128 x 128 blocks, FP32 or power-of-two scales ----------------------------


def test_block128_reduces_to_mxfp8_when_the_scale_is_a_power_of_two():
    # Every 32-block holds one element of magnitude 448 * 2^k (the 128 x 128 block's amax), so
    # amax / 448 = 2^k exactly: both scale modes give s = 2^k, and the MXFP8 rule gives every
    # 32-block the same scale 2^k (floor(log2(448 * 2^k)) - 8 = k). Codes must then equal the
    # (independently pinned) MXFP8 rowwise quantizer's.
    g = np.random.default_rng(31)
    for k in (-9, 0, 5):
        x = torch.from_numpy(g.normal(0.0, 2.0 ** k * 40.0, (128, 256)))
        x = torch.clamp(x, -448 * 2.0 ** k, 448 * 2.0 ** k)
        x[:, ::32] = 448 * 2.0 ** k * torch.sign(torch.from_numpy(g.normal(size=(128, 8))))
        xb = x.to(torch.bfloat16)
        q_mx, s_mx = oracle.quantize_rowwise(xb)
        assert np.all(s_mx == 127 + k)
        for pow2 in (False, True):
            q, s = oracle.quantize_block128(xb, pow2)
            assert np.all(s == np.float32(2.0 ** k))
            assert np.array_equal(q, q_mx)


def test_block128_scale_properties():
    g = np.random.default_rng(32)
    x = torch.from_numpy(g.normal(0.0, 0.02, (256, 384)) * np.exp(g.normal(0.0, 2.0, (256, 384)))).to(torch.bfloat16)
    xd = x.double().numpy()
    q32, s32 = oracle.quantize_block128(x, False)
    q2, s2 = oracle.quantize_block128(x, True)
    dec = np.array([oracle.e4m3_decode(c) for c in range(256)])
    for i in range(2):
        for j in range(3):
            blk = xd[128 * i:128 * (i + 1), 128 * j:128 * (j + 1)]
            amax = np.abs(blk).max()
            a = np.unravel_index(np.abs(blk).argmax(), blk.shape)
            # FP32 scale: the amax element lands on +-448.
            assert abs(dec[q32[128 * i + a[0], 128 * j + a[1]]]) == 448.0
            assert s32[i, j] == np.float32(np.float32(amax) / np.float32(448.0))
            # Power-of-two scale: the power of two that brackets amax / 448 from above.
            e = math.log2(float(s2[i, j]))
            assert e == int(e) and s2[i, j] >= s32[i, j] and s2[i, j] < 2 * s32[i, j]
            assert 224.0 <= abs(dec[q2[128 * i + a[0], 128 * j + a[1]]]) <= 448.0
    # The two grids differ on generic weights: the gap the FP8-blockwise pairing carries.
    assert np.mean(q32 != q2) > 0.3


def test_block128_special_blocks_and_edges():
    x = torch.zeros((130, 160), dtype=torch.bfloat16)
    x[0, 0] = float("nan")                       # block (0, 0): NaN policy
    x[129, 150] = -3.0                           # edge block (1, 1): 2 x 32 elements
    for pow2 in (False, True):
        q, s = oracle.quantize_block128(x, pow2)
        assert s.shape == (2, 2) and np.isnan(s[0, 0])
        assert np.all(q[:128, :128] == 0x7F) and s[0, 1] == 1.0 and s[1, 0] == 1.0
        assert np.all(q[:128, 128:] == 0) and np.all(q[128:, :128] == 0)
        q_edge, s_edge = oracle.quantize_block128(x[128:, 128:].contiguous(), pow2)
        assert s[1, 1] == s_edge[0, 0] and np.array_equal(q[128:, 128:], q_edge)
