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
// One CTA per 128 x 128 tile (persistent over tiles); thread t owns the 32-blocks (row t / 4,
// K-block t % 4) and (row 64 + t / 4, same K-block), as in the MXFP8 rowwise kernel; the tile's
// amax is a warp-shuffle and shared-memory maximum. Must not be compiled with fast-math: the
// divisions are IEEE.
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

__global__ void __launch_bounds__(kQThreads) quantize_block128_kernel(const __grid_constant__ Block128Args a) {
    __shared__ uint32_t warp_max[kQThreads / 32];
    __shared__ float tile_scale;
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    QTensor T{};
    T.x = a.x;
    T.ldx = a.ldx;
    T.vec32 = a.vec32;
    const int64_t tiles = static_cast<int64_t>(a.tiles_m) * a.tiles_k;
    for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x) {
        const int mt = static_cast<int>(t / a.tiles_k), kt = static_cast<int>(t % a.tiles_k);
        const int64_t col = static_cast<int64_t>(kt) * kQTile + (tid & 3) * 32;
        Block32 b[2];
        bool valid[2];
        uint32_t m = 0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int64_t row = static_cast<int64_t>(mt) * kQTile + h * 64 + (tid >> 2);
            valid[h] = row < a.M && col < a.K;
            load_block(T, row, col, valid[h], b[h]);      // zeros outside the tensor
#pragma unroll
            for (int j = 0; j < 4; ++j)
                m = bf16x2_absmax(m, bf16x2_absmax(bf16x2_absmax(b[h].v[j].x, b[h].v[j].y),
                                                   bf16x2_absmax(b[h].v[j].z, b[h].v[j].w)));
        }
        m &= 0x7FFF7FFFu;
        uint32_t mm = max(m & 0xFFFFu, m >> 16);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mm = max(mm, __shfl_xor_sync(0xFFFFFFFFu, mm, o));
        if (lane == 0) warp_max[tid >> 5] = mm;
        __syncthreads();
        if (tid == 0) {
            uint32_t v = 0;
#pragma unroll
            for (int w = 0; w < kQThreads / 32; ++w) v = max(v, warp_max[w]);
            float s;
            if (v >= 0x7F80u) {
                s = __int_as_float(0x7FC00000);           // NaN or Inf in the block
            } else if (v == 0u) {
                s = 1.0f;
            } else {
                s = __uint_as_float(v << 16) / 448.0f;    // IEEE single division
                if (a.pow2) s = pow2_at_least(s);
            }
            tile_scale = s;
            a.scales[static_cast<int64_t>(mt) * a.tiles_k + kt] = s;
        }
        __syncthreads();
        const float s = tile_scale;
        const bool special = !(s == s);
        const uint64_t one2 = 0x3F8000003F800000ull;       // {1, 1}: the codes' only rounding is the cvt
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            if (!valid[h]) continue;
            const int64_t row = static_cast<int64_t>(mt) * kQTile + h * 64 + (tid >> 2);
            uint32_t o[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t w[4] = {b[h].v[j].x, b[h].v[j].y, b[h].v[j].z, b[h].v[j].w};
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    const uint32_t w0 = w[2 * p], w1 = w[2 * p + 1];
                    if (!special) {
                        const float f0 = __uint_as_float(w0 << 16) / s, f1 = __uint_as_float(w0 & 0xFFFF0000u) / s;
                        const float f2 = __uint_as_float(w1 << 16) / s, f3 = __uint_as_float(w1 & 0xFFFF0000u) / s;
                        o[2 * j + p] = enc_quad(__float_as_uint(f0), __float_as_uint(f1), __float_as_uint(f2),
                                                __float_as_uint(f3), one2);
                    } else {
                        o[2 * j + p] = 0x7F7F7F7Fu | ((w0 >> 8) & 0x80u) | ((w0 >> 16) & 0x8000u) |
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
        __syncthreads();                                   // warp_max / tile_scale reused next tile
    }
}

}  // namespace mx
