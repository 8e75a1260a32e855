// MXFP8 quantizer (rowwise and/or columnwise, optionally writing the tensor-core scale layout
// directly) and the standalone scale rearrangement.
//
// The paper ("End-to-End MXFP8 Reinforcement Learning on Blackwell", Figure 1 and Table 6) has the
// learner quantize BF16 masters and activations, then rearrange the E8M0 scales ("scale
// rearrangement", 2.6 ms per micro-batch, more than the 2.2 ms of quantization). Here both happen in
// one HBM pass: a CTA owns a 128 x 128 BF16 tile, whose rowwise scales (128 rows x 4 K-blocks) and
// columnwise scales (128 K-rows x 4 M-blocks) are each exactly one 512-byte block of the
// tensor-core scale layout, so the swizzled scales leave the CTA as one coalesced 512-byte store.
//
// Rule (OCP MX v1.0, which the paper's "E8M0 scales keep only the exponent", Table 10 F6, refers
// to): per 32-block, e = floor(log2 amax) - 8 clamped to [-127, 127], scale byte e + 127;
// elements RNE(x * 2^-e) saturated to +-448 in E4M3. For BF16 input, floor(log2 amax) is the
// biased exponent field minus 127, so the scale byte is max(E_amax - 8, 0), computed on integer
// bits. x * 2^-e is exact in fp32, and one cvt.rn.satfinite rounds it. Blocks holding NaN or Inf
// get scale 0xFF and element bytes sign|0x7F.
//
// This file must not be compiled with flush-to-zero: BF16 subnormal inputs scaled by 2^127 are
// normal E4M3 values.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace mx {

constexpr int kQTile = 128;          // rows and columns of a quantizer tile
constexpr int kQThreads = 256;

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Packs RNE-saturated E4M3 codes of (hi, lo) into 16 bits: lo in bits 0-7, hi in bits 8-15.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float hi, float lo) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Scale byte from the largest BF16 magnitude bits of a block (0 .. 0x7FFF).
__device__ __forceinline__ uint32_t scale_byte_from_amax(uint32_t amax_bits) {
    if (amax_bits >= 0x7F80u) return 0xFFu;            // Inf or NaN in the block
    const int E = static_cast<int>(amax_bits >> 7);    // biased exponent of amax (0 for subnormal/zero)
    return static_cast<uint32_t>(E > 8 ? E - 8 : 0);
}

// 2^-e as an fp32 for scale byte s = e + 127 (s <= 246 for BF16 input): biased exponent 254 - s.
__device__ __forceinline__ float inv_scale(uint32_t s) {
    return s <= 246u ? __uint_as_float((254u - s) << 23) : 1.0f;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Two BF16 (one word) -> two E4M3 codes (16 bits), given the block's scale byte and 2^-e.
__device__ __forceinline__ uint32_t encode_word(uint32_t w, uint32_t s, float inv) {
    if (s == 0xFFu) return 0x7F7Fu | ((w >> 8) & 0x80u) | (((w >> 24) & 0x80u) << 8);
    return cvt_e4m3x2(bf16_hi(w) * inv, bf16_lo(w) * inv);
}

struct QuantArgs {
    const uint16_t* x;
    int64_t M, K, ldx;
    uint8_t* q_row;
    uint8_t* s_row;
    uint8_t* q_col;
    uint8_t* s_col;
    int swz_row, swz_col;
    int64_t tiles_m, tiles_k, tiles;
};

template <bool ROW, bool COL>
__global__ void __launch_bounds__(kQThreads) quantize_kernel(const QuantArgs a) {
    __shared__ __align__(16) uint4 tile[COL ? kQTile * 16 : 1];   // 128 rows x 16 chunks of 8 BF16
    __shared__ __align__(16) uint8_t atom_row[512];
    __shared__ __align__(16) uint8_t atom_col[512];

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int64_t kblocks = a.K / 32;

    uint4 cur[8], nxt[8];
    auto load_tile = [&](uint4 (&v)[8], int64_t t) {
        const int64_t m0 = (t / a.tiles_k) * kQTile, k0 = (t % a.tiles_k) * kQTile;
        const int cc = tid & 15;
#pragma unroll
        for (int it = 0; it < 8; ++it) {
            const int row = it * 16 + (tid >> 4);
            const int64_t m = m0 + row, k = k0 + cc * 8;
            if (m < a.M && k < a.K)
                v[it] = ld_stream_v4(a.x + m * a.ldx + k);
            else
                v[it] = make_uint4(0, 0, 0, 0);
        }
    };

    int64_t t = blockIdx.x;
    if (t < a.tiles) load_tile(cur, t);
    for (; t < a.tiles; t += gridDim.x) {
        const int64_t tn = t + gridDim.x;
        if (tn < a.tiles) load_tile(nxt, tn);
        const int64_t mt = t / a.tiles_k, kt = t % a.tiles_k;
        const int64_t m0 = mt * kQTile, k0 = kt * kQTile;

        if constexpr (COL) {
#pragma unroll
            for (int it = 0; it < 8; ++it) tile[(it * 16 + (tid >> 4)) * 16 + (tid & 15)] = cur[it];
        }

        if constexpr (ROW) {
            // Four consecutive lanes hold one 32-block (8 BF16 each) of one row.
            const int cc = tid & 15;
#pragma unroll
            for (int it = 0; it < 8; ++it) {
                const int row = it * 16 + (tid >> 4);
                const int64_t m = m0 + row, k = k0 + cc * 8;
                const bool valid = (m < a.M) && (k < a.K);
                const uint4 v = cur[it];
                uint32_t mx = max_u16x2(max_u16x2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
                                        max_u16x2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu));
                mx = max(mx & 0xFFFFu, mx >> 16);
                mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
                mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 2));
                const uint32_t s = scale_byte_from_amax(mx);
                const float inv = inv_scale(s);
                if (valid) {
                    uint2 o;
                    o.x = encode_word(v.x, s, inv) | (encode_word(v.y, s, inv) << 16);
                    o.y = encode_word(v.z, s, inv) | (encode_word(v.w, s, inv) << 16);
                    *reinterpret_cast<uint2*>(a.q_row + m * a.K + k) = o;
                }
                if ((lane & 3) == 0)
                    atom_row[(row & 31) * 16 + (row >> 5) * 4 + (cc >> 2)] = valid ? static_cast<uint8_t>(s) : 0;
            }
        }

        if constexpr (COL) {
            __syncthreads();
            // Warp w: M-block (w >> 1) of 32 rows, chunks (w & 1) * 8 .. +7; lane = chunk (low 3
            // bits) + 8 * (8-row group inside the M-block). Each lane reads 8 rows x 8 columns.
            const int chunk = (warp & 1) * 8 + (lane & 7);
            const int rgq = lane >> 3;
            const int mb = warp >> 1;
            uint4 r[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) r[i] = tile[(mb * 32 + rgq * 8 + i) * 16 + chunk];
            uint32_t m4[4];
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                uint32_t mm = 0;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint32_t word = (w == 0 ? r[i].x : w == 1 ? r[i].y : w == 2 ? r[i].z : r[i].w);
                    mm = max_u16x2(mm, word & 0x7FFF7FFFu);
                }
                mm = max_u16x2(mm, __shfl_xor_sync(0xFFFFFFFFu, mm, 8));
                mm = max_u16x2(mm, __shfl_xor_sync(0xFFFFFFFFu, mm, 16));
                m4[w] = mm;
            }
            const int64_t kcol0 = k0 + chunk * 8;
            const int64_t mrow0 = m0 + mb * 32;
            const bool valid = (kcol0 < a.K) && (mrow0 < a.M);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int w = j >> 1, h = j & 1;
                const uint32_t amax = h ? (m4[w] >> 16) : (m4[w] & 0xFFFFu);
                const uint32_t s = scale_byte_from_amax(amax);
                const float inv = inv_scale(s);
                uint32_t e[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint32_t word = (w == 0 ? r[i].x : w == 1 ? r[i].y : w == 2 ? r[i].z : r[i].w);
                    e[i] = h ? (word >> 16) : (word & 0xFFFFu);      // BF16 bits of (row i, column j)
                }
                uint2 o;
                if (s == 0xFFu) {
                    o.x = 0x7F7F7F7Fu | ((e[0] >> 8) & 0x80u) | (((e[1] >> 8) & 0x80u) << 8) |
                          (((e[2] >> 8) & 0x80u) << 16) | (((e[3] >> 8) & 0x80u) << 24);
                    o.y = 0x7F7F7F7Fu | ((e[4] >> 8) & 0x80u) | (((e[5] >> 8) & 0x80u) << 8) |
                          (((e[6] >> 8) & 0x80u) << 16) | (((e[7] >> 8) & 0x80u) << 24);
                } else {
                    o.x = cvt_e4m3x2(__uint_as_float(e[1] << 16) * inv, __uint_as_float(e[0] << 16) * inv) |
                          (cvt_e4m3x2(__uint_as_float(e[3] << 16) * inv, __uint_as_float(e[2] << 16) * inv) << 16);
                    o.y = cvt_e4m3x2(__uint_as_float(e[5] << 16) * inv, __uint_as_float(e[4] << 16) * inv) |
                          (cvt_e4m3x2(__uint_as_float(e[7] << 16) * inv, __uint_as_float(e[6] << 16) * inv) << 16);
                }
                if (valid) *reinterpret_cast<uint2*>(a.q_col + (kcol0 + j) * a.M + mrow0 + rgq * 8) = o;
                if (rgq == 0) {
                    const int kk = chunk * 8 + j;   // K-row inside the tile
                    atom_col[(kk & 31) * 16 + (kk >> 5) * 4 + mb] = valid ? static_cast<uint8_t>(s) : 0;
                }
            }
        }

        __syncthreads();
        // Scale output: one 512-byte block of the tensor-core layout per direction, or raw bytes.
        if constexpr (ROW) {
            if (a.swz_row) {
                if (tid < 32)
                    reinterpret_cast<uint4*>(a.s_row + (mt * a.tiles_k + kt) * 512)[tid] =
                        reinterpret_cast<const uint4*>(atom_row)[tid];
            } else if (tid < kQTile) {
                const int64_t m = m0 + tid;
                const int64_t nb = (kblocks - kt * 4 < 4 ? kblocks - kt * 4 : 4);
                if (m < a.M)
                    for (int b = 0; b < nb; ++b)
                        a.s_row[m * kblocks + kt * 4 + b] = atom_row[(tid & 31) * 16 + (tid >> 5) * 4 + b];
            }
        }
        if constexpr (COL) {
            const int64_t mblocks = a.M / 32;
            const int u = tid - 128;
            if (a.swz_col) {
                if (u >= 0 && u < 32)
                    reinterpret_cast<uint4*>(a.s_col + (kt * a.tiles_m + mt) * 512)[u] =
                        reinterpret_cast<const uint4*>(atom_col)[u];
            } else if (u >= 0) {
                const int64_t k = k0 + u;
                const int64_t nb = (mblocks - mt * 4 < 4 ? mblocks - mt * 4 : 4);
                if (k < a.K)
                    for (int b = 0; b < nb; ++b)
                        a.s_col[k * mblocks + mt * 4 + b] = atom_col[(u & 31) * 16 + (u >> 5) * 4 + b];
            }
        }
        __syncthreads();
#pragma unroll
        for (int it = 0; it < 8; ++it) cur[it] = nxt[it];
    }
}

// ---- standalone scale rearrangement ---------------------------------------------------------

constexpr int kSwzMaxGroups = 128;   // groups per launch; more groups are split over launches

struct SwizzleArgs {
    const uint8_t* s;         // raw scales [rows, kblocks]
    uint8_t* out;             // swizzled output (this launch's groups start at out)
    int64_t kblocks, ctiles;  // ctiles = ceil(kblocks / 4)
    int ngroups;
    int64_t src_row[kSwzMaxGroups];     // first raw row of each group
    int64_t rows[kSwzMaxGroups];        // rows in each group
    int64_t block_start[kSwzMaxGroups + 1];   // first output 512-byte block of each group
};

// One warp per 512-byte output block; lane l assembles 16 bytes: rows l, l+32, l+64, l+96 of the
// block's 128-row tile, 4 K-blocks each.
__global__ void __launch_bounds__(256) swizzle_kernel(const __grid_constant__ SwizzleArgs a) {
    const int lane = threadIdx.x & 31;
    const int64_t nblocks = a.block_start[a.ngroups];
    for (int64_t blk = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; blk < nblocks;
         blk += (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5) {
        int g = 0;
        while (g + 1 < a.ngroups && a.block_start[g + 1] <= blk) ++g;
        const int64_t local = blk - a.block_start[g];
        const int64_t rt = local / a.ctiles, ct = local % a.ctiles;
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t r = rt * 128 + lane + 32 * j;
            uint32_t word = 0;
            if (r < a.rows[g]) {
                const uint8_t* src = a.s + (a.src_row[g] + r) * a.kblocks + ct * 4;
                const int64_t nb = (a.kblocks - ct * 4 < 4 ? a.kblocks - ct * 4 : 4);
                for (int b = 0; b < nb; ++b) word |= static_cast<uint32_t>(src[b]) << (8 * b);
            }
            w[j] = word;
        }
        reinterpret_cast<uint4*>(a.out + blk * 512)[lane] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

}  // namespace mx
