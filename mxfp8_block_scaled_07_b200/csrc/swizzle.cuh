// Standalone scale rearrangement into the tensor-core scale layout (the paper's "scale
// rearrangement", Table 6; the interleaved scale copy a backend derives, Table 10 F3), for one
// matrix or for groups of rows each padded to 128 rows (the A-operand layout of the grouped GEMM).
#pragma once
#include <cstdint>

namespace mx {

constexpr int kSwzMaxGroups = 128;   // groups per launch; more groups are split over launches

struct SwizzleArgs {
    const uint8_t* s;         // raw scales [rows, kblocks]
    uint8_t* out;             // swizzled output (this launch's groups start at out)
    int64_t kblocks, ctiles;  // ctiles = ceil(kblocks / 4)
    int ngroups;
    int word_loads;           // kblocks % 4 == 0 and s 4-byte aligned: a row's 4 bytes in one load
    int64_t src_row[kSwzMaxGroups];     // first raw row of each group
    int64_t rows[kSwzMaxGroups];        // rows in each group
    int64_t block_start[kSwzMaxGroups + 1];   // first output 512-byte block of each group
};

// Group of output block `blk`: the largest g with block_start[g] <= blk.
__device__ __forceinline__ int swz_group(const SwizzleArgs& a, int64_t blk) {
    int lo = 0, hi = a.ngroups - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.block_start[mid] <= blk) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ uint4 ld_nc_u4(const uint8_t* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// QUAD == false: one warp per 512-byte output block; lane l assembles 16 bytes, the 4 K-blocks of
// rows l, l+32, l+64, l+96 of the block's 128-row tile (one 32-bit load per row when word_loads,
// else byte loads). QUAD == true (kblocks % 16 == 0, s 16-byte aligned): one warp per 4 consecutive
// blocks of a row tile; lane l loads 16 bytes (16 K-blocks) of each of its 4 rows and writes its
// 16-byte piece of all 4 blocks.
template <bool QUAD>
__global__ void __launch_bounds__(256) swizzle_kernel(const __grid_constant__ SwizzleArgs a) {
    constexpr int kPer = QUAD ? 4 : 1;
    const int lane = threadIdx.x & 31;
    const int64_t nunits = a.block_start[a.ngroups] / kPer;
    for (int64_t u = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; u < nunits;
         u += (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5) {
        const int64_t blk = u * kPer;
        const int g = swz_group(a, blk);
        const int64_t local = blk - a.block_start[g];
        const int64_t rt = local / a.ctiles, ct = local % a.ctiles;
        if constexpr (QUAD) {
            uint4 v[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int64_t r = rt * 128 + lane + 32 * j;
                v[j] = r < a.rows[g] ? ld_nc_u4(a.s + (a.src_row[g] + r) * a.kblocks + ct * 4) : make_uint4(0, 0, 0, 0);
            }
            uint4* o = reinterpret_cast<uint4*>(a.out + blk * 512) + lane;
            o[0] = make_uint4(v[0].x, v[1].x, v[2].x, v[3].x);
            o[32] = make_uint4(v[0].y, v[1].y, v[2].y, v[3].y);
            o[64] = make_uint4(v[0].z, v[1].z, v[2].z, v[3].z);
            o[96] = make_uint4(v[0].w, v[1].w, v[2].w, v[3].w);
        } else {
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int64_t r = rt * 128 + lane + 32 * j;
                uint32_t word = 0;
                if (r < a.rows[g]) {
                    const uint8_t* src = a.s + (a.src_row[g] + r) * a.kblocks + ct * 4;
                    if (a.word_loads) {
                        word = __ldg(reinterpret_cast<const uint32_t*>(src));
                    } else {
                        const int64_t nb = (a.kblocks - ct * 4 < 4 ? a.kblocks - ct * 4 : 4);
                        for (int b = 0; b < nb; ++b) word |= static_cast<uint32_t>(src[b]) << (8 * b);
                    }
                }
                w[j] = word;
            }
            reinterpret_cast<uint4*>(a.out + blk * 512)[lane] = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

}  // namespace mx
