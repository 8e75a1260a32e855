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
// TMEM columns (x 128 lanes, 32-bit): accumulator 0 = [0, 256), accumulator 1 = [240, 496) (the two
// share [240, 256)), scale slot = [496, 508): A scales 4 columns, B scales 8 columns.
constexpr uint32_t kAcc1Col = 240;
constexpr uint32_t kOvlCol = 240;
constexpr uint32_t kSfCol = 496;

constexpr int kSmemA = 0;
constexpr int kSmemB = kSmemA + kStages * kABytes;
constexpr int kSmemSfa = kSmemB + kStages * kBBytes;
constexpr int kSmemSfb = kSmemSfa + kStages * kSfaBytes;
constexpr int kStageBytes = 32 * 128;  // epilogue staging per warp: 32 rows x 128 bytes (TMA-store box)
constexpr int kSmemStage = kSmemSfb + kStages * kSfbBytes;            // 1024-aligned
constexpr int kSmemBar = kSmemStage + 4 * kStageBytes;
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
    int tma_store;      // output written by TMA from swizzled shared-memory staging (tmap_c valid)
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
                   const __grid_constant__ CUtensorMap tmap_c, const GemmArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kSmemBar);
    uint64_t* empty = full + kStages;
    uint64_t* tmem_full = empty + kStages;
    uint64_t* ovl_free = tmem_full + 1;     // epilogue has drained the shared accumulator columns
    uint64_t* drain = ovl_free + 1;
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
        mbar_init(ovl_free, 4 * 32);
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
        // Tile j accumulates into TMEM columns [acc_j, acc_j + 256): acc_j = 0 for even j, 240 for odd
        // j. The two accumulators share columns 240-255, which the epilogue reads first; tile j starts
        // as soon as those of tile j-1 are drained (by then the epilogue has finished tile j-2). The
        // scale blocks go to one TMEM slot (columns 496-507): tcgen05 operations issued by one thread
        // execute in order, so a copy never overtakes the MMAs that read the previous contents.
        int stage = 0;
        uint32_t phase = 0, ovl_phase = 0;
        bool ok = true;
        const uint32_t sfa_t = tmem_base + kSfCol;
        const uint32_t sfb_t = sfa_t + 4;
        int j = 0;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++j) {
            if (j > 0) {
                if (!mbar_wait(ovl_free, ovl_phase, abort, a.err, a.timeout_ns)) { ok = false; break; }
                ovl_phase ^= 1u;
            }
            tc_fence_after();
            const uint32_t acc = tmem_base + ((j & 1) ? kAcc1Col : 0u);
            for (int kb = 0; kb < a.nkb; ++kb) {
                if (!mbar_wait(&full[stage], phase, abort, a.err, a.timeout_ns)) { ok = false; break; }
                tc_fence_after();
                if (lane == 0) {
                    tc_cp_32x128b_warpx4(sfa_t, sdesc_scale_block(smem_u32(smem + kSmemSfa + stage * kSfaBytes)));
                    tc_cp_32x128b_warpx4(sfb_t, sdesc_scale_block(smem_u32(smem + kSmemSfb + stage * kSfbBytes)));
                    tc_cp_32x128b_warpx4(sfb_t + 4,
                                         sdesc_scale_block(smem_u32(smem + kSmemSfb + stage * kSfbBytes + 512)));
                    const uint64_t adesc = sdesc_kmajor_sw128(smem_u32(smem + kSmemA + stage * kABytes));
                    const uint64_t bdesc = sdesc_kmajor_sw128(smem_u32(smem + kSmemB + stage * kBBytes));
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        // K-step k: +32 bytes inside the 128-byte swizzled rows; scale byte k.
                        tc_mma_mxf8(acc, adesc + 2u * k, bdesc + 2u * k, idesc_mxf8_e4m3(kBM, kBN, k),
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
        }
        // Every MMA issued by this thread has completed once `drain` fires.
        if (lane == 0) tc_commit(drain);
        __syncwarp();
        mbar_wait_drain(drain, 0, a.timeout_ns);
    } else {
        // ---------------- epilogue ----------------
        // Warp w reads TMEM lanes 32 * (w % 4) .. +31 (rows of the tile). The accumulator is released
        // as soon as its last columns are in registers; rows leave through a per-warp swizzled
        // staging buffer and a TMA store (32 rows x 128 bytes per store), or, for rows that a TMA
        // box must not cover (a grouped tile's rows past its group) or unaligned outputs, through
        // direct masked stores.
        const int q = warp & 3;
        const int row_local = q * 32 + lane;
        uint8_t* stage = smem + kSmemStage + (warp - 2) * kStageBytes;
        const uint32_t stage_row = smem_u32(stage) + lane * 128;
        const uint32_t swz = static_cast<uint32_t>(lane & 7);
        uint32_t full_phase = 0;
        int j = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++j) {
            const Tile T = decode_tile<GROUPED>(t, a, off, pm);
            if (!mbar_wait(tmem_full, full_phase, abort, a.err, a.timeout_ns)) break;
            full_phase ^= 1u;
            tc_fence_after();
            const int warp_rows = min(32, max(0, T.rows_valid - q * 32));
            const bool use_tma = a.tma_store && warp_rows > 0 && (!GROUPED || warp_rows == 32);
            const bool row_ok = row_local < T.rows_valid;
            const int64_t crow = static_cast<int64_t>(T.a_row0) + row_local;
            const uint32_t lanes = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
            const bool acc1 = (j & 1) != 0;
            const uint32_t tq = lanes + (acc1 ? kAcc1Col : 0u);
            // The shared columns first (tile columns 240..255 of accumulator 0, 0..15 of accumulator
            // 1); once every epilogue thread has them, the next tile's MMAs may start.
            uint32_t ov[16];
            tc_ld_32x32b_x16(lanes + kOvlCol, ov);
            tc_wait_ld();
            tc_fence_before();
            mbar_arrive(ovl_free);
            // Writes one 128-byte row piece p (64 BF16 or 32 fp32 columns starting at col0) of this
            // warp's 32 rows.
            auto emit = [&](const uint32_t(&p)[32], int col0, int cols) {
                if (col0 >= a.N) return;
                if (use_tma) {
                    if (lane == 0) bulk_wait_group_read<0>();   // staging buffer no longer read
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        st_shared_v4(stage_row + ((static_cast<uint32_t>(i) ^ swz) << 4), p[4 * i], p[4 * i + 1],
                                     p[4 * i + 2], p[4 * i + 3]);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tmap_c, stage, col0, T.a_row0 + q * 32);
                        bulk_commit_group();
                    }
                } else if (row_ok) {
                    const int ncols = min(cols, a.N - col0);
                    if (ncols == cols && a.vec_store) {
                        uint4* d4 = reinterpret_cast<uint4*>(static_cast<uint8_t*>(a.c) +
                                                             (crow * a.ldc + col0) * (a.out_bf16 ? 2 : 4));
#pragma unroll
                        for (int i = 0; i < 8; ++i) d4[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
                    } else if (a.out_bf16) {
                        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(a.c) + crow * a.ldc + col0;
#pragma unroll
                        for (int i = 0; i < 64; ++i)
                            if (i < ncols) dst[i] = __ushort_as_bfloat16(static_cast<unsigned short>(p[i >> 1] >> (16 * (i & 1))));
                    } else {
                        float* dst = reinterpret_cast<float*>(a.c) + crow * a.ldc + col0;
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (i < ncols) dst[i] = __uint_as_float(p[i]);
                    }
                }
            };
            // Columns [c * 16, c * 16 + 32) for even c: from the shared columns already in `ov` where
            // they fall there, else from TMEM.
            auto fetch32 = [&](int c, uint32_t(&p)[32]) {
                const bool lo_shared = acc1 && c == 0;          // tile columns 0..15 of accumulator 1
                const bool hi_shared = !acc1 && c == 14;        // tile columns 240..255 of accumulator 0
                if (lo_shared || hi_shared) {
                    uint32_t r[16];
                    tc_ld_32x32b_x16(tq + (lo_shared ? 16u : 224u), r);
                    tc_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        p[i] = lo_shared ? ov[i] : r[i];
                        p[16 + i] = lo_shared ? r[i] : ov[i];
                    }
                } else {
                    tc_ld_32x32b_x32(tq + c * 16, p);
                    tc_wait_ld();
                }
            };
            if (a.out_bf16) {
                uint32_t pk[4][32];                          // the row's 256 columns, packed BF16
#pragma unroll
                for (int c = 0; c < 16; c += 2) {
                    uint32_t r[32];
                    fetch32(c, r);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
                        pk[c >> 2][((c >> 1) & 1) * 16 + i] = *reinterpret_cast<const uint32_t*>(&h);
                    }
                }
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) emit(pk[ch], T.n0 + ch * 64, 64);
            } else {
#pragma unroll
                for (int c = 0; c < 16; c += 2) {
                    uint32_t p[32];
                    fetch32(c, p);
                    emit(p, T.n0 + c * 16, 32);
                }
            }
        }
        if (lane == 0) bulk_wait_group<0>();                 // every TMA store of this warp complete
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace mx
