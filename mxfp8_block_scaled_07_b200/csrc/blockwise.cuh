// FP8 blockwise quantization: E4M3 codes with one scale per 128 x 128 block of a BF16 weight.
//
// "End-to-End MXFP8 Reinforcement Learning on Blackwell" (Table 1) pairs an FP8-blockwise learner
// with an FP8-blockwise sampler whose scales differ on SM100: the learner's are powers of two (its
// GEMMs run as MXFP8, whose E8M0 scales keep only the exponent; Table 10 F6), the sampler's are
// FP32. The two grids of the same weights therefore differ; this kernel produces either one so
// the gap can be measured against the MXFP8 path's shared grid.
//
// Rule: amax = max |x| over the block; FP32 scales s = fl32(amax / 448), codes
// RNE_E4M3(fl32(x / s)) saturated to +-448 (both divisions IEEE single precision); power-of-two
// scales s = the smallest power of two >= fl32(amax / 448), codes RNE_E4M3(x / s). An all-zero
// block takes s = 1; a block holding NaN or Inf takes s = NaN and codes sign | 0x7F.
//
// A persistent grid, each CTA a contiguous range of 128 x 128 tiles; thread t owns the 32-blocks
// (row t / 4, K-block t % 4) and (row 64 + t / 4, same K-block). The tile's amax is a warp-shuffle
// maximum, then one barrier over double-buffered per-warp maxima that every thread reduces itself.
// With power-of-two scales x / s is the exact product x * (1 / s) whenever 1 / s is a finite fp32
// power of two, so those codes come from the MXFP8 encoder's multiply; that form is HBM-bound and
// keeps the next tile's loads in flight while it encodes the current one (2 CTAs per SM, as the
// MXFP8 rowwise kernel). FP32 scales keep the IEEE division per element; that form is bound by the
// divisions and runs without the prefetch at 4 CTAs per SM, for more warps. Must not be compiled
// with fast-math: the divisions are IEEE.
#pragma once
#include <cstdint>

#include "quantize.cuh"

namespace mx {

struct Block128Args {
    const uint16_t* x;
    uint8_t* q;
    float* scales;
    int64_t M, K, ldx;
    int tiles_m, tiles_k;
    int pow2;               // power-of-two scales (else FP32)
    int vec32;              // x rows and q rows 32-byte aligned: 256-bit loads and stores
};

// The smallest power of two >= v (v > 0, finite).
__device__ __forceinline__ float pow2_at_least(float v) {
    const int e = ilogbf(v);
    const float p = ldexpf(1.0f, e);
    return p == v ? p : ldexpf(1.0f, e + 1);
}

// Scale of a tile from the largest magnitude bits of its elements (0 .. 0x7FFF).
__device__ __forceinline__ float block128_scale(uint32_t v, bool pow2) {
    if (v >= 0x7F80u) return __int_as_float(0x7FC00000);   // NaN or Inf in the block
    if (v == 0u) return 1.0f;
    const float s = __uint_as_float(v << 16) / 448.0f;       // IEEE single division
    return pow2 ? pow2_at_least(s) : s;
}

template <bool POW2>
__global__ void __launch_bounds__(kQThreads, POW2 ? 2 : 4)
    quantize_block128_kernel(const __grid_constant__ Block128Args a) {
    __shared__ uint32_t warp_max[2][kQThreads / 32];
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    QTensor T{};
    T.x = a.x;
    T.ldx = a.ldx;
    T.vec32 = a.vec32;
    const int64_t tiles = static_cast<int64_t>(a.tiles_m) * a.tiles_k;
    // POW2: a contiguous range of tiles per CTA; FP32: tiles dealt round-robin (neighbouring CTAs
    // on neighbouring tiles), measured faster for the division-bound form.
    const int64_t per = POW2 ? (tiles + gridDim.x - 1) / gridDim.x : 1;
    const int64_t stride = POW2 ? 1 : gridDim.x;
    const int64_t t_begin = static_cast<int64_t>(blockIdx.x) * per;
    const int64_t t_end = POW2 ? min(tiles, t_begin + per) : tiles;
    const int64_t colo = (tid & 3) * 32;
    auto load_tile = [&](int64_t t, Block32 (&b)[2]) {
        const int64_t mt = t / a.tiles_k, kt = t % a.tiles_k;
        const int64_t col = kt * kQTile + colo;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int64_t row = mt * kQTile + h * 64 + (tid >> 2);
            load_block(T, row, col, row < a.M && col < a.K, b[h]);      // zeros outside the tensor
        }
    };
    Block32 cur[2], nxt[2];
    if (POW2 && t_begin < t_end) load_tile(t_begin, cur);
    int it = 0;
    for (int64_t t = t_begin; t < t_end; t += stride, ++it) {
        if constexpr (POW2) {
            if (t + 1 < t_end) load_tile(t + 1, nxt);
        } else {
            load_tile(t, cur);
        }
        const int p = it & 1;
        const int64_t mt = t / a.tiles_k, kt = t % a.tiles_k;
        const int64_t col = kt * kQTile + colo;
        uint32_t m = 0;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int j = 0; j < 4; ++j)
                m = bf16x2_absmax(m, bf16x2_absmax(bf16x2_absmax(cur[h].v[j].x, cur[h].v[j].y),
                                                   bf16x2_absmax(cur[h].v[j].z, cur[h].v[j].w)));
        m &= 0x7FFF7FFFu;
        uint32_t mm = max(m & 0xFFFFu, m >> 16);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mm = max(mm, __shfl_xor_sync(0xFFFFFFFFu, mm, o));
        if (lane == 0) warp_max[p][tid >> 5] = mm;
        __syncthreads();
        uint32_t v = 0;
#pragma unroll
        for (int w = 0; w < kQThreads / 32; ++w) v = max(v, warp_max[p][w]);
        const float s = block128_scale(v, POW2);
        if (tid == 0) a.scales[mt * a.tiles_k + kt] = s;
        const bool special = !(s == s);
        // Power-of-two scale with a finite reciprocal: x / s == x * (1 / s) exactly.
        const bool mul = POW2 && !special && s >= 0x1p-126f;
        const uint32_t inv = __float_as_uint(1.0f / s);
        const uint64_t inv2 = (static_cast<uint64_t>(inv) << 32) | inv;
        const uint64_t one2 = 0x3F8000003F800000ull;       // {1, 1}: the codes' only rounding is the cvt
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int64_t row = mt * kQTile + h * 64 + (tid >> 2);
            if (!(row < a.M && col < a.K)) continue;
            uint32_t o[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t w[4] = {cur[h].v[j].x, cur[h].v[j].y, cur[h].v[j].z, cur[h].v[j].w};
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const uint32_t w0 = w[2 * q], w1 = w[2 * q + 1];
                    if (mul) {
                        o[2 * j + q] = enc_words(w0, w1, inv2);
                    } else if (!special) {
                        const float f0 = __uint_as_float(w0 << 16) / s, f1 = __uint_as_float(w0 & 0xFFFF0000u) / s;
                        const float f2 = __uint_as_float(w1 << 16) / s, f3 = __uint_as_float(w1 & 0xFFFF0000u) / s;
                        o[2 * j + q] = enc_quad(__float_as_uint(f0), __float_as_uint(f1), __float_as_uint(f2),
                                                __float_as_uint(f3), one2);
                    } else {
                        o[2 * j + q] = 0x7F7F7F7Fu | ((w0 >> 8) & 0x80u) | ((w0 >> 16) & 0x8000u) |
                                       ((w1 << 8) & 0x800000u) | (w1 & 0x80000000u);
                    }
                }
            }
            uint8_t* dst = a.q + row * a.K + col;
            const uint4 lo = make_uint4(o[0], o[1], o[2], o[3]);
            const uint4 hi = make_uint4(o[4], o[5], o[6], o[7]);
            if (a.vec32) {
                st_v8(dst, lo, hi);
            } else {
                reinterpret_cast<uint4*>(dst)[0] = lo;
                reinterpret_cast<uint4*>(dst)[1] = hi;
            }
        }
        if constexpr (POW2) {
            cur[0] = nxt[0];
            cur[1] = nxt[1];
        }
    }
}

}  // namespace mx
