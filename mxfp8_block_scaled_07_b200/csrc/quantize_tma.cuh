// MXFP8 quantizer with TMA-staged tiles: rowwise, columnwise or both, optionally writing the
// tensor-core scale layout directly, over one tensor or a list of tensors in one launch.
//
// Same rule, outputs and tile decomposition as quantize.cuh ("End-to-End MXFP8 Reinforcement
// Learning on Blackwell", Figure 1 and Table 6: the learner's MXFP8 quantization and the scale
// rearrangement, here one HBM pass). What differs is how the BF16 tile reaches the threads: each
// CTA keeps a ring of kQtStages 128 x 128 BF16 tiles (32 KB each) in shared memory, filled by 2-D
// TMA tensor loads of this GPU's own memory (128-byte swizzle) that run kQtStages tiles ahead of
// the compute, so a CTA's loads stay in flight while it quantizes, and a small tensor's tiles are
// all requested at once. Both passes read the tile from shared memory:
//   - rowwise: warp w takes 32 consecutive rows (32 (w % 4) + lane) and K-block 2 (w / 4) + pass;
//     the eight lanes of a quarter-warp read the same 16-byte chunk of eight consecutive rows,
//     which the swizzle spreads over all 32 banks;
//   - columnwise: thread t takes the column pair 2 (t % 64), +1 over the 32-row M-block t / 64, one
//     32-bit word per row (32 consecutive words of one 128-byte row per warp: conflict-free).
// Out-of-range rows and columns of a ragged tile arrive as zeros (TMA fill) and are masked on
// store; a half tile lying wholly past K is not loaded at all.
//
// The wait for a stage is bounded (globaltimer deadline, error bit 1); after an expired wait the
// CTA waits for its copies still in flight (at least 1 s) and returns.
//
// This file must not be compiled with flush-to-zero (see quantize.cuh).
#pragma once
#include <cstdint>

#include "ptx.cuh"
#include "quantize.cuh"

namespace mx {

constexpr int kQtStages = 3;
constexpr int kQtHalfBytes = 128 * 128;            // 128 rows x 64 BF16 (one TMA box)
constexpr int kQtStageBytes = 2 * kQtHalfBytes;    // one 128 x 128 BF16 tile
constexpr int kQtMaxTensors = 160;                 // tensor maps + descriptors < 32 KB of parameters
// Dynamic shared memory: stages (1024-aligned for the swizzle), barriers, two pairs of scale blocks.
constexpr int kQtSmemBytes = kQtStages * kQtStageBytes + 64 + 2 * 2 * 512 + 1024;

struct QtTensor {
    uint8_t* q_row;
    uint8_t* s_row;
    uint8_t* q_col;
    uint8_t* s_col;
    int64_t tile_start;       // first tile of this tensor in the launch's tile space
    int32_t M, K;
    int32_t tiles_m, tiles_k;
    int32_t vec32;            // q_row 32-byte aligned: 256-bit stores
    int32_t col_vec32;        // q_col 32-byte aligned
};

template <int NT>
struct QuantTmaArgs {
    CUtensorMap map[NT];      // BF16 [M, K] of tensor i: boxes of 64 columns x 128 rows, 128-byte swizzle
    QtTensor t[NT];
    int n;
    int swz;
    int64_t total_tiles;
    uint32_t* err;
    uint64_t timeout_ns;
};

__device__ __forceinline__ void tma_load_2d(uint32_t smem_dst, const CUtensorMap* map, uint32_t bar, int32_t c0,
                                            int32_t c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
        "[%2];" ::"r"(smem_dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}

struct QtTile {
    int i;                    // tensor
    int mt, kt;
    int64_t m0, k0;
    bool full;                // the whole 128 x 128 tile lies inside the tensor
};

template <int NT>
__device__ __forceinline__ QtTile qt_decode(const QuantTmaArgs<NT>& a, int64_t t) {
    int i = 0;
    if constexpr (NT > 1) {
        int lo = 0, hi = a.n - 1;    // largest i with tile_start <= t
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (a.t[mid].tile_start <= t) lo = mid; else hi = mid - 1;
        }
        i = lo;
    }
    const QtTensor& T = a.t[i];
    const int64_t local = t - T.tile_start;
    QtTile r;
    r.i = i;
    r.mt = static_cast<int>(local / T.tiles_k);
    r.kt = static_cast<int>(local % T.tiles_k);
    r.m0 = static_cast<int64_t>(r.mt) * kQTile;
    r.k0 = static_cast<int64_t>(r.kt) * kQTile;
    r.full = (r.m0 + kQTile <= T.M) && (r.k0 + kQTile <= T.K);
    return r;
}

// The tile after r in the launch's tile space (row-major within a tensor, tensors in order).
template <int NT>
__device__ __forceinline__ void qt_next(const QuantTmaArgs<NT>& a, QtTile& r) {
    if (++r.kt == a.t[r.i].tiles_k) {
        r.kt = 0;
        if (++r.mt == a.t[r.i].tiles_m) {
            r.mt = 0;
            ++r.i;
        }
    }
    if (r.i < a.n) {
        const QtTensor& T = a.t[r.i];
        r.m0 = static_cast<int64_t>(r.mt) * kQTile;
        r.k0 = static_cast<int64_t>(r.kt) * kQTile;
        r.full = (r.m0 + kQTile <= T.M) && (r.k0 + kQTile <= T.K);
    }
}

// Requests tile r into stage buffer `dst` (one thread): one box per 64-column half that overlaps K.
template <int NT>
__device__ __forceinline__ void qt_issue(const QuantTmaArgs<NT>& a, const QtTile& r, uint32_t dst, uint64_t* bar) {
    const bool second = r.k0 + 64 < a.t[r.i].K;
    mbar_arrive_expect_tx(bar, second ? kQtStageBytes : kQtHalfBytes);
    const uint32_t b = smem_u32(bar);
    tma_load_2d(dst, &a.map[r.i], b, static_cast<int32_t>(r.k0), static_cast<int32_t>(r.m0));
    if (second) tma_load_2d(dst + kQtHalfBytes, &a.map[r.i], b, static_cast<int32_t>(r.k0 + 64), static_cast<int32_t>(r.m0));
}

// Byte offset of 16-byte chunk c (0..7) of row r inside a 128-byte-swizzled half tile.
__device__ __forceinline__ uint32_t qt_chunk(int r, int c) {
    return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

template <bool ROW, bool COL, int NT>
__global__ void __launch_bounds__(kQThreads, 2) quantize_tma_kernel(const __grid_constant__ QuantTmaArgs<NT> a) {
    extern __shared__ uint8_t qt_smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(qt_smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t stages_s = smem_u32(smem);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kQtStages * kQtStageBytes);
    volatile int* abort = reinterpret_cast<volatile int*>(full + kQtStages);
    uint8_t* atoms = smem + kQtStages * kQtStageBytes + 64;     // [2 buffers][row, col][512]
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;

    const int64_t total = a.total_tiles;
    const int64_t t_begin = static_cast<int64_t>(blockIdx.x) * total / gridDim.x;
    const int64_t t_end = static_cast<int64_t>(blockIdx.x + 1) * total / gridDim.x;
    if (tid == 0) {
        for (int s = 0; s < kQtStages; ++s) mbar_init(&full[s], 1);
        *abort = 0;
        fence_barrier_init();
    }
    __syncthreads();
    // Tiles are walked incrementally: every thread steps `rc` through its CTA's range, and thread 0
    // also steps `ri`, the next tile to request (kQtStages ahead).
    QtTile rc, ri;
    if (t_begin < t_end) rc = ri = qt_decode(a, t_begin);
    if (tid == 0)
        for (int s = 0; s < kQtStages && t_begin + s < t_end; ++s) {
            qt_issue(a, ri, stages_s + s * kQtStageBytes, &full[s]);
            qt_next(a, ri);
        }

    int64_t t = t_begin;
    for (int j = 0; t < t_end; ++t, ++j, qt_next(a, rc)) {
        const int s = j % kQtStages;
        const bool ok = mbar_wait(&full[s], static_cast<uint32_t>(j / kQtStages) & 1u, abort, a.err, a.timeout_ns);
        if (__syncthreads_or(!ok)) break;
        const QtTensor& T = a.t[rc.i];
        const uint32_t st = stages_s + s * kQtStageBytes;
        uint8_t* atom_row = atoms + (j & 1) * 1024;
        uint8_t* atom_col = atom_row + 512;

        if constexpr (ROW) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int r = (warp & 3) * 32 + lane;            // row inside the tile
                const int kb = (warp >> 2) * 2 + h;              // K-block inside the tile
                const uint32_t base = st + (kb >> 1) * kQtHalfBytes;
                Block32 b;
#pragma unroll
                for (int c = 0; c < 4; ++c) b.v[c] = ld_shared_v4(base + qt_chunk(r, (kb & 1) * 4 + c));
                const int64_t row = rc.m0 + r;
                const int64_t col = rc.k0 + kb * 32;
                const bool valid = rc.full || (row < T.M && col < T.K);
                uint32_t m = bf16x2_absmax(bf16x2_absmax(b.v[0].x, b.v[0].y), bf16x2_absmax(b.v[0].z, b.v[0].w));
#pragma unroll
                for (int c = 1; c < 4; ++c)
                    m = bf16x2_absmax(m, bf16x2_absmax(bf16x2_absmax(b.v[c].x, b.v[c].y),
                                                       bf16x2_absmax(b.v[c].z, b.v[c].w)));
                m &= 0x7FFF7FFFu;
                const uint32_t sc = scale_byte_from_amax(max(m & 0xFFFFu, m >> 16));
                uint4 o0, o1;
                uint2 e;
                e = encode_chunk(b.v[0], sc);
                o0.x = e.x; o0.y = e.y;
                e = encode_chunk(b.v[1], sc);
                o0.z = e.x; o0.w = e.y;
                e = encode_chunk(b.v[2], sc);
                o1.x = e.x; o1.y = e.y;
                e = encode_chunk(b.v[3], sc);
                o1.z = e.x; o1.w = e.y;
                if (valid) {
                    uint8_t* q = T.q_row + row * T.K + col;
                    if (T.vec32) {
                        st_v8(q, o0, o1);
                    } else {
                        reinterpret_cast<uint4*>(q)[0] = o0;
                        reinterpret_cast<uint4*>(q)[1] = o1;
                    }
                }
                atom_row[(r & 31) * 16 + (r >> 5) * 4 + kb] = valid ? static_cast<uint8_t>(sc) : 0;
            }
        }
        if constexpr (COL) {
            const int cp = tid & 63;                     // column pair: tile columns 2 cp, 2 cp + 1
            const int mb = tid >> 6;                     // 32-row M-block
            const uint32_t base = st + (cp >> 5) * kQtHalfBytes + (cp & 3) * 4;
            const int cc = (cp & 31) >> 2;               // 16-byte chunk inside the half's 128-byte row
            uint32_t w[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) w[i] = ld_shared_u32(base + qt_chunk(mb * 32 + i, cc));
            const uint32_t m = col_pair_absmax(w);
            const int64_t kc = rc.k0 + 2 * cp;           // K-row of the transposed copy (low halves)
            const int64_t mr = rc.m0 + 32 * mb;
            const bool mok = rc.full || mr < T.M;        // M % 32 == 0: a block is all in or all out
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const uint32_t sc = scale_byte_from_amax(hh ? (m >> 16) : (m & 0xFFFFu));
                const bool ok2 = mok && (rc.full || kc + hh < T.K);
                uint32_t o[8];
                encode_col32(w, sc, hh != 0, o);
                if (ok2) {
                    uint8_t* q = T.q_col + (kc + hh) * T.M + mr;
                    const uint4 lo = make_uint4(o[0], o[1], o[2], o[3]);
                    const uint4 hi4 = make_uint4(o[4], o[5], o[6], o[7]);
                    if (T.col_vec32) {
                        st_v8(q, lo, hi4);
                    } else {
                        reinterpret_cast<uint4*>(q)[0] = lo;
                        reinterpret_cast<uint4*>(q)[1] = hi4;
                    }
                }
                const int kk = 2 * cp + hh;              // K-row inside the tile
                atom_col[(kk & 31) * 16 + (kk >> 5) * 4 + mb] = ok2 ? static_cast<uint8_t>(sc) : 0;
            }
        }
        __syncthreads();     // stage s read by every thread; this tile's scale blocks complete
        if (tid == 0 && t + kQtStages < t_end) {
            qt_issue(a, ri, st, &full[s]);
            qt_next(a, ri);
        }
        // Scale output: one 512-byte block of the tensor-core layout per direction, or raw bytes. The
        // other pair of atom buffers takes the next tile, so no second barrier is needed here.
        if constexpr (ROW) {
            if (a.swz) {
                if (tid < 32)
                    reinterpret_cast<uint4*>(T.s_row + (static_cast<int64_t>(rc.mt) * T.tiles_k + rc.kt) * 512)[tid] =
                        reinterpret_cast<const uint4*>(atom_row)[tid];
            } else if (tid < kQTile) {
                const int64_t kblocks = T.K / 32;
                const int64_t m_ = rc.m0 + tid;
                const int64_t nb = (kblocks - rc.kt * 4 < 4 ? kblocks - rc.kt * 4 : 4);
                if (m_ < T.M)
                    for (int q = 0; q < nb; ++q)
                        T.s_row[m_ * kblocks + rc.kt * 4 + q] = atom_row[(tid & 31) * 16 + (tid >> 5) * 4 + q];
            }
        }
        if constexpr (COL) {
            const int64_t mblocks = T.M / 32;
            const int u = tid - 128;
            if (a.swz) {
                if (u >= 0 && u < 32)
                    reinterpret_cast<uint4*>(T.s_col + (static_cast<int64_t>(rc.kt) * T.tiles_m + rc.mt) * 512)[u] =
                        reinterpret_cast<const uint4*>(atom_col)[u];
            } else if (u >= 0) {
                const int64_t k = rc.k0 + u;
                const int64_t nb = (mblocks - rc.mt * 4 < 4 ? mblocks - rc.mt * 4 : 4);
                if (k < T.K)
                    for (int q = 0; q < nb; ++q)
                        T.s_col[k * mblocks + rc.mt * 4 + q] = atom_col[(u & 31) * 16 + (u >> 5) * 4 + q];
            }
        }
    }
    // After an expired wait: the copies requested for tiles t .. min(t + stages, t_end) - 1 may still
    // be in flight into this CTA's shared memory; wait for them before the CTA exits.
    if (t < t_end && tid == 0) {
        const int j0 = static_cast<int>(t - t_begin);
        for (int j = j0; j < j0 + kQtStages && t_begin + j < t_end; ++j)
            mbar_wait_drain(&full[j % kQtStages], static_cast<uint32_t>(j / kQtStages) & 1u, a.timeout_ns);
    }
}

}  // namespace mx
