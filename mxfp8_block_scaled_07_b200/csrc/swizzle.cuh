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
