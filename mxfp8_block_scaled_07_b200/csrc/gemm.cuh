// Block-scaled MXFP8 GEMM on the 5th-generation tensor cores (tcgen05, kind::mxf8f6f4.block_scale).
//
// C[m, n] = sum_k A[m, k] * 2^(ea[m, k/32]) * B[n, k] * 2^(eb[n, k/32]), fp32 accumulation in TMEM,
// fp32 or BF16 (RNE) output. Both operands are K-major E4M3 ([rows, K]); their E8M0 scales arrive
// in the tensor-core scale layout (128 x 4 blocks of 512 bytes), which is what the MMA reads from
// TMEM. This is the learner's and sampler's MXFP8 linear of "End-to-End MXFP8 Reinforcement Learning
// on Blackwell" (Table 6: GEMM 20.4 ms BF16 vs 13.3 ms MXFP8 per micro-batch; Table 2: dense
// Qwen3-8B and the 128-expert Qwen3-30B-A3B MoE, whose expert GEMMs run grouped).
//
// Design (one CTA per SM, persistent, static tile schedule, warp-specialized):
//   warp 0     TMA producer: A tile 128 x 128 B, B tile 256 x 128 B (128-byte swizzle), and the
//              512-byte scale blocks (1 for A, 2 for B) by bulk copy, into a 4-stage ring;
//   warp 1     TMEM owner and MMA issuer: per stage, tcgen05.cp of the scale blocks into TMEM,
//              then 4 MMAs of 128 x 256 x 32 (one per 32-K block, selecting its scale byte);
//   warps 2-5  epilogue: tcgen05.ld of the 128 x 256 fp32 accumulator (warp w reads TMEM lanes
//              32 * (w % 4) ..), convert, store to global.
// Every mbarrier wait is bounded (globaltimer deadline); on expiry the kernel records an error
// bit, stops all roles, drains its in-flight copies and MMAs, frees TMEM and returns.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace mx {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 128;            // bytes of K per stage (= one 128-byte swizzle row)
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK;  // 16 KB
constexpr int kBBytes = kBN * kBK;  // 32 KB
constexpr int kSfaBytes = 512;
constexpr int kSfbBytes = 1024;
constexpr int kGemmThreads = 192;
constexpr int kMaxGroups = 1024;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCols = kBN;  // fp32 accumulator: 256 TMEM columns x 128 lanes

constexpr int kSmemA = 0;
constexpr int kSmemB = kSmemA + kStages * kABytes;
constexpr int kSmemSfa = kSmemB + kStages * kBBytes;
constexpr int kSmemSfb = kSmemSfa + kStages * kSfaBytes;
constexpr int kSmemBar = kSmemSfb + kStages * kSfbBytes;
constexpr int kSmemMisc = kSmemBar + (2 * kStages + 3) * 8;
constexpr int kSmemGroups = (kSmemMisc + 16 + 15) / 16 * 16;
constexpr int kGemmSmemDense = kSmemGroups + 1024;                                  // + alignment slack
constexpr int kGemmSmemGrouped = kSmemGroups + 2 * (kMaxGroups + 1) * 4 + 1024;

struct GemmArgs {
    const uint8_t* sfa;
    const uint8_t* sfb;
    void* c;
    int64_t ldc;
    int M;              // dense: rows of A; grouped: total rows
    int N, K;
    int nkb;            // ceil(K / 128)
    int tiles_m, tiles_n;
    int out_bf16;
    int vec_store;      // output rows 16-byte aligned: full 32-column chunks use 16-byte stores
    int G;
    int n_rowtiles;     // ceil(N / 128): scale row-tiles of one B operand
    const int32_t* row_offsets;
    uint32_t* err;
    uint64_t timeout_ns;
};

struct Tile {
    int a_row0;         // first A row (TMA coordinate)
    int rows_valid;     // rows of C this tile owns
    int b_row0;         // first B row (TMA coordinate)
    int n0;             // first output column
    int sfa_tile;       // 128-row tile index into A's scale layout
    int sfb_tile;       // 128-row tile index into B's scale layout
};

template <bool GROUPED>
__device__ __forceinline__ Tile decode_tile(int t, const GemmArgs& a, const int32_t* off, const int32_t* pm) {
    Tile T;
    if constexpr (!GROUPED) {
        const int mt = t % a.tiles_m, nt = t / a.tiles_m;
        T.a_row0 = mt * kBM;
        T.rows_valid = min(kBM, a.M - T.a_row0);
        T.n0 = nt * kBN;
        T.b_row0 = T.n0;
        T.sfa_tile = mt;
        T.sfb_tile = T.n0 / 128;
    } else {
        const int mtg = t / a.tiles_n, nt = t % a.tiles_n;
        int lo = 0, hi = a.G - 1;      // largest g with pm[g] <= mtg
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (pm[mid] <= mtg) lo = mid; else hi = mid - 1;
        }
        const int g = lo;
        T.a_row0 = off[g] + (mtg - pm[g]) * kBM;
        T.rows_valid = min(kBM, off[g + 1] - T.a_row0);
        T.n0 = nt * kBN;
        T.b_row0 = g * a.N + T.n0;
        T.sfa_tile = mtg;
        T.sfb_tile = g * a.n_rowtiles + T.n0 / 128;
    }
    return T;
}

template <bool GROUPED>
__global__ void __launch_bounds__(kGemmThreads, 1)
    mx_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                   const GemmArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kSmemBar);
    uint64_t* empty = full + kStages;
    uint64_t* tmem_full = empty + kStages;
    uint64_t* tmem_empty = tmem_full + 1;
    uint64_t* drain = tmem_empty + 1;
    uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(smem + kSmemMisc);
    volatile int* abort = reinterpret_cast<volatile int*>(smem + kSmemMisc + 4);
    int* total_tiles = reinterpret_cast<int*>(smem + kSmemMisc + 8);
    int32_t* off = reinterpret_cast<int32_t*>(smem + kSmemGroups);
    int32_t* pm = off + (kMaxGroups + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(tmem_full, 1);
        mbar_init(tmem_empty, 4 * 32);
        mbar_init(drain, 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmap_a);
        prefetch_tensormap(&tmap_b);
    }
    if (warp == 1) {
        tmem_alloc(tmem_base_slot, kTmemCols);
        tmem_relinquish();
    }
    if constexpr (GROUPED) {
        for (int g = threadIdx.x; g <= a.G; g += blockDim.x) off[g] = a.row_offsets[g];
        __syncthreads();
        if (threadIdx.x == 0) {
            bool ok = off[0] == 0 && off[a.G] == a.M;
            int acc = 0;
            for (int g = 0; g < a.G; ++g) {
                pm[g] = acc;
                const int n = off[g + 1] - off[g];
                if (n < 0) ok = false;
                acc += n > 0 ? (n + kBM - 1) / kBM : 0;
            }
            pm[a.G] = acc;
            if (!ok) atomicOr(a.err, kErrBadOffsets);
            *total_tiles = ok ? acc * a.tiles_n : 0;
        }
    } else {
        if (threadIdx.x == 0) *total_tiles = a.tiles_m * a.tiles_n;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_base_slot;
    const int tiles = *total_tiles;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        int stage = 0;
        uint32_t phase = 0;
        int issued = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
            const Tile T = decode_tile<GROUPED>(t, a, off, pm);
            const bool sfb1 = T.n0 + 128 < a.N;
            const uint32_t bytes = kABytes + kBBytes + kSfaBytes + (sfb1 ? 1024u : 512u);
            for (int kb = 0; kb < a.nkb; ++kb) {
                if (!mbar_wait(&empty[stage], phase ^ 1u, abort, a.err, a.timeout_ns)) { ok = false; break; }
                if (lane == 0) {
                    mbar_arrive_expect_tx(&full[stage], bytes);
                    tma_load_2d(smem + kSmemA + stage * kABytes, &tmap_a, &full[stage], kb * kBK, T.a_row0);
                    tma_load_2d(smem + kSmemB + stage * kBBytes, &tmap_b, &full[stage], kb * kBK, T.b_row0);
                    bulk_load(smem + kSmemSfa + stage * kSfaBytes,
                              a.sfa + (static_cast<int64_t>(T.sfa_tile) * a.nkb + kb) * 512, 512, &full[stage]);
                    bulk_load(smem + kSmemSfb + stage * kSfbBytes,
                              a.sfb + (static_cast<int64_t>(T.sfb_tile) * a.nkb + kb) * 512, 512, &full[stage]);
                    if (sfb1)
                        bulk_load(smem + kSmemSfb + stage * kSfbBytes + 512,
                                  a.sfb + (static_cast<int64_t>(T.sfb_tile + 1) * a.nkb + kb) * 512, 512,
                                  &full[stage]);
                }
                __syncwarp();
                ++issued;
                if (++stage == kStages) { stage = 0; phase ^= 1u; }
            }
        }
        if (!ok) {
            // Wait for the copies still in flight (the last min(issued, kStages) fills).
            int s = stage;
            uint32_t p = phase;
            for (int i = 0; i < min(issued, kStages); ++i) {
                if (--s < 0) { s = kStages - 1; p ^= 1u; }
                mbar_wait_drain(&full[s], p, a.timeout_ns);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        int stage = 0;
        uint32_t phase = 0, acc_phase = 0;
        bool ok = true;
        const uint32_t sfa_base = tmem_base + kAccCols;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
            if (!mbar_wait(tmem_empty, acc_phase ^ 1u, abort, a.err, a.timeout_ns)) { ok = false; break; }
            tc_fence_after();
            for (int kb = 0; kb < a.nkb; ++kb) {
                if (!mbar_wait(&full[stage], phase, abort, a.err, a.timeout_ns)) { ok = false; break; }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t sfa_t = sfa_base + stage * 16;
                    const uint32_t sfb_t = sfa_t + 4;
                    tc_cp_32x128b_warpx4(sfa_t, sdesc_scale_block(smem_u32(smem + kSmemSfa + stage * kSfaBytes)));
                    tc_cp_32x128b_warpx4(sfb_t, sdesc_scale_block(smem_u32(smem + kSmemSfb + stage * kSfbBytes)));
                    tc_cp_32x128b_warpx4(sfb_t + 4,
                                         sdesc_scale_block(smem_u32(smem + kSmemSfb + stage * kSfbBytes + 512)));
                    const uint64_t adesc = sdesc_kmajor_sw128(smem_u32(smem + kSmemA + stage * kABytes));
                    const uint64_t bdesc = sdesc_kmajor_sw128(smem_u32(smem + kSmemB + stage * kBBytes));
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        // K-step k: +32 bytes inside the 128-byte swizzled rows; scale byte k.
                        tc_mma_mxf8(tmem_base, adesc + 2u * k, bdesc + 2u * k, idesc_mxf8_e4m3(kBM, kBN, k),
                                    sfa_t | (static_cast<uint32_t>(k) << 30), sfb_t | (static_cast<uint32_t>(k) << 30),
                                    (kb | k) != 0 ? 1u : 0u);
                    }
                    tc_commit(&empty[stage]);
                }
                __syncwarp();
                if (++stage == kStages) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
            if (lane == 0) tc_commit(tmem_full);
            __syncwarp();
            acc_phase ^= 1u;
        }
        // Every MMA issued by this thread has completed once `drain` fires.
        if (lane == 0) tc_commit(drain);
        __syncwarp();
        mbar_wait_drain(drain, 0, a.timeout_ns);
    } else {
        // ---------------- epilogue ----------------
        const int q = warp & 3;                 // TMEM lane quarter this warp may read
        const int row_local = q * 32 + lane;
        uint32_t acc_phase = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
            const Tile T = decode_tile<GROUPED>(t, a, off, pm);
            if (!mbar_wait(tmem_full, acc_phase, abort, a.err, a.timeout_ns)) break;
            tc_fence_after();
            const bool row_ok = row_local < T.rows_valid;
            const int64_t crow = static_cast<int64_t>(T.a_row0) + row_local;
#pragma unroll 1
            for (int c = 0; c < kBN / 32; ++c) {
                uint32_t r[32];
                tc_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + c * 32, r);
                tc_wait_ld();
                const int col0 = T.n0 + c * 32;
                if (!row_ok || col0 >= a.N) continue;
                const int ncols = min(32, a.N - col0);
                if (a.out_bf16) {
                    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(a.c) + crow * a.ldc + col0;
                    if (ncols == 32 && a.vec_store) {
                        uint32_t p[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const __nv_bfloat162 h =
                                __floats2bfloat162_rn(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
                            p[i] = *reinterpret_cast<const uint32_t*>(&h);
                        }
                        uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
                        for (int i = 0; i < 4; ++i) d4[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (i < ncols) dst[i] = __float2bfloat16_rn(__uint_as_float(r[i]));
                    }
                } else {
                    float* dst = reinterpret_cast<float*>(a.c) + crow * a.ldc + col0;
                    if (ncols == 32 && a.vec_store) {
                        uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
                        for (int i = 0; i < 8; ++i) d4[i] = make_uint4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (i < ncols) dst[i] = __uint_as_float(r[i]);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(tmem_empty);
            acc_phase ^= 1u;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace mx
