// Block-scaled MXFP8 GEMM on the 5th-generation tensor cores (tcgen05, kind::mxf8f6f4.block_scale).
//
// C[m, n] = sum_k A[m, k] * 2^(ea[m, k/32]) * B[n, k] * 2^(eb[n, k/32]), fp32 accumulation in TMEM,
// fp32 or BF16 (RNE) output. Both operands are K-major E4M3 ([rows, K]); their E8M0 scales arrive
// in the tensor-core scale layout (128 x 4 blocks of 512 bytes), which is what the MMA reads from
// TMEM. This is the learner's and sampler's MXFP8 linear of "End-to-End MXFP8 Reinforcement Learning
// on Blackwell" (Table 6: GEMM 20.4 ms BF16 vs 13.3 ms MXFP8 per micro-batch; Table 2: dense
// Qwen3-8B and the 128-expert Qwen3-30B-A3B MoE, whose expert GEMMs run grouped).
//
// Two kernels, both persistent with a static tile schedule and warp specialization:
//
//   mx_gemm_pair_kernel (default): a cluster of 2 CTAs on two SMs computes a 256 x 256 tile with
//     tcgen05.mma.cta_group::2 (M = 256, N = 256). Each CTA loads its own 128 rows of A, half of B's
//     256 rows and the full 256-row B scale tile; the leader CTA issues the scale copies and MMAs for
//     both. Per SM this halves B traffic and the scale-copy work per FLOP against one CTA alone.
//   mx_gemm_kernel: one CTA computes a 128 x 256 tile with cta_group::1 MMAs.
//
// The pair kernel's EPI = 1 instantiation (grouped only) replaces the C store with the MoE expert
// activation and the down projection's MXFP8 quantization (epilogue_swiglu_tile).
//
// Roles (320 threads): warp 0 TMA producer (A/B tiles with the 128-byte swizzle, scale blocks);
// warp 1 TMEM owner and MMA issuer; warps 2-9 epilogue in two groups of four (warp w reads TMEM
// lanes 32 * (w % 4); group (w - 2) / 4 drains one accumulator, i.e. every other tile).
// TMEM: two accumulators overlapping in 16 columns ([0, 256) and [240, 496)) and one scale slot
// ([496, 508)): the epilogue drains the shared columns first, so the next tile's MMAs start while
// the rest of the previous tile is still being read out. tcgen05 operations issued by one thread
// execute in order, so a scale copy never overtakes the MMAs that read the slot's previous contents.
// The epilogue writes through per-warp swizzled staging and coalesced 16-byte stores. Tiles walk M
// first, or N first when A is the larger operand, so the smaller operand stays in L2.
//
// Every mbarrier wait is bounded (globaltimer deadline); on expiry the kernel records an error bit,
// stops all roles, drains its in-flight copies and MMAs, frees TMEM and returns. No load uses
// cluster multicast.
#pragma once
#include <cstdint>
#include <type_traits>

#include "ptx.cuh"
#include "quantize.cuh"    // the E4M3 encoding helpers, shared with the fused SwiGLU epilogue

namespace mx {

constexpr int kBM = 128;            // rows of A per CTA
constexpr int kBN = 256;            // columns of C per tile
constexpr int kBK = 128;            // bytes of K per stage (= one 128-byte swizzle row)
constexpr int kSfaBytes = 512;
constexpr int kSfbBytes = 1024;
constexpr int kEpiWarps = 8;          // two groups of four, one warp per TMEM lane quadrant each
constexpr int kGemmThreads = 64 + 32 * kEpiWarps;
constexpr int kMaxGroups = 1024;
constexpr uint32_t kTmemCols = 512;
// TMEM columns (x 128 lanes, 32-bit): accumulator 0 = [0, 256), accumulator 1 = [240, 496) (the two
// share [240, 256)), scale slot = [496, 508): A scales 4 columns, B scales 8 columns.
constexpr uint32_t kAcc1Col = 240;
constexpr uint32_t kOvlCol = 240;
constexpr uint32_t kSfCol = 496;
constexpr int kStageBytes = 32 * 128;  // epilogue staging per warp: 32 rows x 128 bytes

// Shared-memory layout of one kernel configuration. B_ROWS: rows of B per CTA and stage.
template <int STAGES, int B_ROWS, int GROUP_ARRAYS>
struct GemmSmem {
    static constexpr int kStages = STAGES;
    static constexpr int kA = 0;
    static constexpr int kB = kA + STAGES * kBM * kBK;
    static constexpr int kSfa = kB + STAGES * B_ROWS * kBK;
    static constexpr int kSfb = kSfa + STAGES * kSfaBytes;
    static constexpr int kStage = (kSfb + STAGES * kSfbBytes + 1023) / 1024 * 1024;
    static_assert(kA % 1024 == 0 && kB % 1024 == 0, "swizzled operand buffers 1024-aligned");
    static constexpr int kBar = kStage + kEpiWarps * kStageBytes;
    static constexpr int kMisc = kBar + (2 * STAGES + 6) * 8;
    static constexpr int kGroups = (kMisc + 16 + 15) / 16 * 16;
    static constexpr int kBytes = kGroups + GROUP_ARRAYS * (kMaxGroups + 1) * 4 + 1024;   // + alignment slack
};
using Smem1Dense = GemmSmem<3, kBN, 0>;                    // single-CTA kernel
using Smem1Grouped = GemmSmem<3, kBN, 2>;
using SmemPairDense = GemmSmem<5, kBN / 2, 0>;             // pair kernel
using SmemPairGrouped = GemmSmem<5, kBN / 2, 3>;
constexpr int kGemmSmemDense = Smem1Dense::kBytes;
constexpr int kGemmSmemGrouped = Smem1Grouped::kBytes;
constexpr int kGemmPairSmemDense = SmemPairDense::kBytes;
constexpr int kGemmPairSmemGrouped = SmemPairGrouped::kBytes;
static_assert(kGemmPairSmemDense <= 232448 && kGemmPairSmemGrouped <= 232448 && kGemmSmemGrouped <= 232448 &&
                  kGemmSmemDense <= 232448,
              "shared memory per CTA");

struct GemmArgs {
    const uint8_t* sfa;
    const uint8_t* sfb;
    void* c;
    int64_t ldc;
    int M;              // dense: rows of A; grouped: total rows
    int N, K;
    int nkb;            // ceil(K / 128)
    int tiles_m;        // dense: row tiles (128 rows single-CTA, 256 rows pair)
    int tiles_n;        // 256-column tiles
    int sfa_tiles;      // 128-row tiles in A's scale layout (dense), for clamping
    int out_bf16;
    int vec_store;      // output rows 16-byte aligned: full 16-byte chunks use 16-byte stores
    int G;
    int n_fast;         // dense: consecutive tiles step along N (B re-read from L2, A streamed once)
    int n_rowtiles;     // ceil(N / 128): scale row-tiles of one B operand
    const int32_t* row_offsets;
    uint32_t* err;
    uint64_t timeout_ns;
    // Fused SwiGLU + MXFP8 epilogue (grouped gate_up GEMM): the quantized activation [M, n_inter],
    // its scales in the grouped tensor-core layout (hs_ctiles = n_inter / 128 blocks per 128 rows).
    uint8_t* hq;
    uint8_t* hs;
    int n_inter;
    int hs_ctiles;
};

// What one CTA does for one tile.
struct Tile {
    int a_row0;         // first A row of this CTA (TMA coordinate; also first C row)
    int rows_valid;     // rows of C this CTA owns in the tile (0..128)
    int b_row0;         // first B row this CTA loads (TMA coordinate)
    int n0;             // first output column
    int sfa_tile;       // 128-row tile index into A's scale layout
    int sfb_tile0;      // 128-row tile indices into B's scale layout (columns n0.., n0 + 128..)
    int sfb_tile1;
};

// Largest g in [0, G) with pm[g] <= x (pm nondecreasing, x < pm[G]).
__device__ __forceinline__ int find_group(const int32_t* pm, int G, int x) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pm[mid] <= x) lo = mid; else hi = mid - 1;
    }
    return lo;
}

template <bool GROUPED>
__device__ __forceinline__ Tile decode_tile1(int t, const GemmArgs& a, const int32_t* off, const int32_t* pm) {
    Tile T;
    if constexpr (!GROUPED) {
        // Tile walk: the smaller operand stays resident in L2 while the larger one streams once.
        const int mt = a.n_fast ? t / a.tiles_n : t % a.tiles_m;
        const int nt = a.n_fast ? t % a.tiles_n : t / a.tiles_m;
        T.a_row0 = mt * kBM;
        T.rows_valid = min(kBM, a.M - T.a_row0);
        T.n0 = nt * kBN;
        T.b_row0 = T.n0;
        T.sfa_tile = mt;
        T.sfb_tile0 = T.n0 / 128;
    } else {
        const int mtg = t / a.tiles_n, nt = t % a.tiles_n;
        const int g = find_group(pm, a.G, mtg);
        T.a_row0 = off[g] + (mtg - pm[g]) * kBM;
        T.rows_valid = min(kBM, off[g + 1] - T.a_row0);
        T.n0 = nt * kBN;
        T.b_row0 = g * a.N + T.n0;
        T.sfa_tile = mtg;
        T.sfb_tile0 = g * a.n_rowtiles + T.n0 / 128;
    }
    T.sfb_tile1 = T.sfb_tile0 + 1;
    return T;
}

// Pair tiles are 256 x 256; CTA `rank` owns rows [128 rank, 128 rank + 128) of the tile and loads B
// rows [n0 + 128 rank, +128). Scale-tile indices past the real ones are clamped to valid memory;
// those rows / columns are never written.
template <bool GROUPED>
__device__ __forceinline__ Tile decode_tile_pair(int t, int rank, const GemmArgs& a, const int32_t* off,
                                                 const int32_t* pm128, const int32_t* pm256) {
    Tile T;
    int sf_last_in_b;
    if constexpr (!GROUPED) {
        // Tile walk: the smaller operand stays resident in L2 while the larger one streams once.
        const int mt = a.n_fast ? t / a.tiles_n : t % a.tiles_m;
        const int nt = a.n_fast ? t % a.tiles_n : t / a.tiles_m;
        T.a_row0 = mt * 2 * kBM + rank * kBM;
        T.rows_valid = max(0, min(kBM, a.M - T.a_row0));
        T.n0 = nt * kBN;
        T.b_row0 = T.n0 + rank * kBM;
        T.sfa_tile = min(2 * mt + rank, a.sfa_tiles - 1);
        T.sfb_tile0 = T.n0 / 128;
        sf_last_in_b = a.n_rowtiles - 1;
    } else {
        const int mtg = t / a.tiles_n, nt = t % a.tiles_n;
        const int g = find_group(pm256, a.G, mtg);
        const int local = mtg - pm256[g];
        T.a_row0 = off[g] + local * 2 * kBM + rank * kBM;
        T.rows_valid = max(0, min(kBM, off[g + 1] - T.a_row0));
        T.n0 = nt * kBN;
        T.b_row0 = g * a.N + T.n0 + rank * kBM;
        T.sfa_tile = min(pm128[g] + 2 * local + rank, pm128[a.G] - 1);
        T.sfb_tile0 = g * a.n_rowtiles + T.n0 / 128;
        sf_last_in_b = g * a.n_rowtiles + a.n_rowtiles - 1;
    }
    T.sfb_tile1 = min(T.sfb_tile0 + 1, sf_last_in_b);
    return T;
}

// Drains the fp32 accumulator of one tile (this warp's 32 TMEM lanes = 32 rows) and writes C.
// Two epilogue groups of four warps (one warp per TMEM lane quadrant) take the tiles in turn, group
// g the tiles in accumulator g, so a group that is still storing one tile never delays the drain of
// the next. The 16 columns the two accumulators share are read first and released with one arrive
// per warp on `ovl_free`; the accumulator itself is released (`acc_empty`) once the last TMEM load
// of the tile has landed, before the last store.
// Rows leave through the warp's swizzled staging box (32 rows x 128 bytes): each lane writes its
// row there, then the warp writes the box out row-contiguous with 16-byte stores (8 lanes per row,
// 4 rows per instruction), masked to the tile's valid rows and to N. The stores go through the
// load/store path, not TMA: TMA stores share the SM's TMA unit with the operand loads and were
// measured to slow those down. Barrier addresses are shared::cluster addresses.
template <bool GROUPED>
__device__ __forceinline__ void epilogue_tile(const GemmArgs& a, const Tile& T, uint32_t tmem_base, bool acc1,
                                              uint8_t* stage, uint32_t ovl_free_addr, uint32_t acc_empty_addr,
                                              int q, int lane) {
    const int warp_rows = min(32, max(0, T.rows_valid - q * 32));
    const int64_t row0 = static_cast<int64_t>(T.a_row0) + q * 32;
    const uint32_t lanes = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const uint32_t tq = lanes + (acc1 ? kAcc1Col : 0u);
    const uint32_t swz = static_cast<uint32_t>(lane & 7);

    uint32_t ov[16];                     // tile columns 240..255 of accumulator 0, 0..15 of accumulator 1
    tc_ld_32x32b_x16(lanes + kOvlCol, ov);
    tc_wait_ld_regs(ov);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive_cluster(ovl_free_addr);

    // Writes one 128-byte row piece p (64 BF16 or 32 fp32 columns starting at col0) of the 32 rows.
    const uint32_t box = smem_u32(stage);
    const int esz = a.out_bf16 ? 2 : 4;
    const int epc = 16 / esz;                            // elements per 16-byte chunk
    auto emit = [&](const uint32_t(&p)[32], int col0) {
        if (col0 >= a.N) return;
        const uint32_t row = box + lane * 128;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            st_shared_v4(row + ((static_cast<uint32_t>(i) ^ swz) << 4), p[4 * i], p[4 * i + 1], p[4 * i + 2],
                         p[4 * i + 3]);
        __syncwarp();
        const int c = lane & 7;                          // this lane's 16-byte chunk of each row
        const int gc = col0 + c * epc;
        const int ncols = min(epc, a.N - gc);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int rr = (lane >> 3) + 4 * i;
            const uint4 v = ld_shared_v4(box + rr * 128 + ((static_cast<uint32_t>(c) ^ (rr & 7)) << 4));
            if (rr < warp_rows && ncols > 0) {
                uint8_t* dst = static_cast<uint8_t*>(a.c) + ((row0 + rr) * a.ldc + gc) * esz;
                if (ncols == epc && a.vec_store) {
                    st_global_v4(dst, v);
                } else {
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                    if (a.out_bf16) {
                        uint16_t* d = reinterpret_cast<uint16_t*>(dst);
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            if (e < ncols) d[e] = static_cast<uint16_t>(w[e >> 1] >> (16 * (e & 1)));
                    } else {
                        uint32_t* d = reinterpret_cast<uint32_t*>(dst);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            if (e < ncols) d[e] = w[e];
                    }
                }
            }
        }
        __syncwarp();                                    // the box is free for the next piece
    };
    // Issues the TMEM loads of tile columns [32 c, 32 c + 32) into p; the shared columns come from `ov`.
    // The caller waits (tc_wait_ld_regs) before reading p.
    auto load32 = [&](int c, uint32_t(&p)[32]) {
        if (acc1 && c == 0) {
            tc_ld_32x32b_x16(tq + 16u, *reinterpret_cast<uint32_t(*)[16]>(&p[16]));
#pragma unroll
            for (int i = 0; i < 16; ++i) p[i] = ov[i];
        } else if (!acc1 && c == 7) {
            tc_ld_32x32b_x16(tq + 224u, *reinterpret_cast<uint32_t(*)[16]>(&p[0]));
#pragma unroll
            for (int i = 0; i < 16; ++i) p[16 + i] = ov[i];
        } else {
            tc_ld_32x32b_x32(tq + 32u * c, p);
        }
    };
    auto release = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc_empty_addr);
    };
    auto pack = [&](const uint32_t(&r)[64], uint32_t(&pk)[32]) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
            pk[i] = *reinterpret_cast<const uint32_t*>(&v);
        }
    };
    if (a.out_bf16) {
        // Four 64-column pieces; the next piece's TMEM loads are in flight while the current one is
        // stored, and the accumulator is released as soon as the last piece is in registers.
        uint32_t raw[64], pa[32], pb[32];
        load32(0, *reinterpret_cast<uint32_t(*)[32]>(&raw[0]));
        load32(1, *reinterpret_cast<uint32_t(*)[32]>(&raw[32]));
        tc_wait_ld_regs(raw);
        pack(raw, pa);
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
            uint32_t(&cur)[32] = (ch & 1) ? pb : pa;
            uint32_t(&nxt)[32] = (ch & 1) ? pa : pb;
            if (ch < 3) {
                load32(2 * ch + 2, *reinterpret_cast<uint32_t(*)[32]>(&raw[0]));
                load32(2 * ch + 3, *reinterpret_cast<uint32_t(*)[32]>(&raw[32]));
            }
            emit(cur, T.n0 + ch * 64);
            if (ch < 3) {
                tc_wait_ld_regs(raw);
                if (ch == 2) release();
                pack(raw, nxt);
            }
        }
    } else {
        // fp32: one 32-column piece at a time, same overlap.
        uint32_t f0[32], f1[32];
        load32(0, f0);
        tc_wait_ld_regs(f0);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint32_t(&cur)[32] = (c & 1) ? f1 : f0;
            uint32_t(&nxt)[32] = (c & 1) ? f0 : f1;
            if (c < 7) load32(c + 1, nxt);
            emit(cur, T.n0 + c * 32);
            if (c < 7) {
                tc_wait_ld_regs(nxt);
                if (c == 6) release();
            }
        }
    }
}

// Fused epilogue of the expert gate_up GEMM: SwiGLU, then the MXFP8 rule, straight into the down
// GEMM's operand. The caller interleaves the weight rows per 128, so tile columns [0, 128) hold the
// gate features f0 .. f0 + 127 and [128, 256) the up features of the same f0 (f0 = 128 * tile
// column index). Each thread (one row) computes h = silu(gate) * up in fp32 from the fp32
// accumulator, 32 features at a time, with CUDA's fast __expf and __fdividef (their error, a few
// ulps growing with |gate|, is part of the stated accuracy); the block's E8M0 scale comes from the fp32 amax (OCP rule:
// e = floor(log2 amax) - 8, clamped at -127, i.e. byte = biased exponent - 8, at least 0; 0xFF when
// the block holds NaN or Inf), the codes from one satfinite E4M3 rounding of h * 2^-e (exact
// power-of-two scaling). 32 code bytes go to hq[row, f0 + 32 b .. ], the 4 scale bytes of the row as
// one word into the grouped tensor-core layout (the CTA's 128 rows are one 128-row scale tile,
// T.sfa_tile, as for the A operand). Rows past the expert's end write zero scale bytes (the
// layout's pad rows) and no codes.
__device__ __forceinline__ void epilogue_swiglu_tile(const GemmArgs& a, const Tile& T, uint32_t tmem_base,
                                                     bool acc1, uint32_t ovl_free_addr, uint32_t acc_empty_addr,
                                                     int q, int lane) {
    const int row_local = q * 32 + lane;
    const bool row_ok = row_local < T.rows_valid;
    const uint32_t lanes = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const uint32_t tq = lanes + (acc1 ? kAcc1Col : 0u);

    uint32_t ov[16];                     // tile columns 240..255 of accumulator 0, 0..15 of accumulator 1
    tc_ld_32x32b_x16(lanes + kOvlCol, ov);
    tc_wait_ld_regs(ov);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive_cluster(ovl_free_addr);

    auto load32 = [&](int c, uint32_t(&p)[32]) {
        if (acc1 && c == 0) {
            tc_ld_32x32b_x16(tq + 16u, *reinterpret_cast<uint32_t(*)[16]>(&p[16]));
#pragma unroll
            for (int i = 0; i < 16; ++i) p[i] = ov[i];
        } else if (!acc1 && c == 7) {
            tc_ld_32x32b_x16(tq + 224u, *reinterpret_cast<uint32_t(*)[16]>(&p[0]));
#pragma unroll
            for (int i = 0; i < 16; ++i) p[16 + i] = ov[i];
        } else {
            tc_ld_32x32b_x32(tq + 32u * c, p);
        }
    };
    const int nt = T.n0 / kBN;
    uint8_t* hrow = a.hq + (static_cast<int64_t>(T.a_row0) + row_local) * a.n_inter + nt * 128;
    uint32_t sbytes = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        uint32_t gw[32], uw[32];
        load32(b, gw);                   // gate features f0 + 32 b ..
        load32(4 + b, uw);               // up features of the same f0 + 32 b ..
        tc_wait_ld_regs(gw, uw);
        if (b == 3) {                    // every TMEM load of the tile has landed
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty_addr);
        }
        float amax = 0.0f;
        bool special = false;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const float g = __uint_as_float(gw[i]);
            const float h = g * __fdividef(1.0f, 1.0f + __expf(-g)) * __uint_as_float(uw[i]);
            special |= !(fabsf(h) <= 3.402823466e38f);   // NaN or Inf
            amax = fmaxf(amax, fabsf(h));
            gw[i] = __float_as_uint(h);
        }
        const uint32_t E = __float_as_uint(amax) >> 23;
        const uint32_t sc = special ? 0xFFu : (E > 8u ? E - 8u : 0u);
        uint32_t o[8];
        if (!special) {
            const uint64_t inv2 = inv_scale2(sc);
#pragma unroll
            for (int k = 0; k < 8; ++k) o[k] = enc_quad(gw[4 * k], gw[4 * k + 1], gw[4 * k + 2], gw[4 * k + 3], inv2);
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                uint32_t r = 0x7F7F7F7Fu;
#pragma unroll
                for (int i = 0; i < 4; ++i) r |= (gw[4 * k + i] >> 31) << (8 * i + 7);
                o[k] = r;
            }
        }
        if (row_ok) {
            uint4* d = reinterpret_cast<uint4*>(hrow + 32 * b);
            d[0] = make_uint4(o[0], o[1], o[2], o[3]);
            d[1] = make_uint4(o[4], o[5], o[6], o[7]);
        }
        sbytes |= (row_ok ? sc : 0u) << (8 * b);
    }
    if (T.rows_valid > 0) {
        const int64_t blk = static_cast<int64_t>(T.sfa_tile) * a.hs_ctiles + nt;
        *reinterpret_cast<uint32_t*>(a.hs + blk * 512 + lane * 16 + q * 4) = sbytes;
    }
}

// Loads the group row offsets into shared memory, checks them and builds the prefix sums of
// row tiles per group (tile_rows = 128: pm128; also 256: pm256 when given). Returns the tile count
// (0 and an error bit when the offsets are invalid). Executed by the whole CTA.
__device__ __forceinline__ int setup_groups(const GemmArgs& a, int32_t* off, int32_t* pm128, int32_t* pm256,
                                            int tiles_n) {
    for (int g = threadIdx.x; g <= a.G; g += blockDim.x) off[g] = a.row_offsets[g];
    __syncthreads();
    __shared__ int total;
    if (threadIdx.x == 0) {
        bool ok = off[0] == 0 && off[a.G] == a.M;
        int acc128 = 0, acc256 = 0;
        for (int g = 0; g < a.G; ++g) {
            pm128[g] = acc128;
            if (pm256) pm256[g] = acc256;
            const int n = off[g + 1] - off[g];
            if (n < 0) ok = false;
            acc128 += n > 0 ? (n + 127) / 128 : 0;
            acc256 += n > 0 ? (n + 255) / 256 : 0;
        }
        pm128[a.G] = acc128;
        if (pm256) pm256[a.G] = acc256;
        if (!ok) atomicOr(a.err, kErrBadOffsets);
        total = ok ? (pm256 ? acc256 : acc128) * tiles_n : 0;
    }
    __syncthreads();
    return total;
}

// ---------------------------------------------------------------------------------------------
// Single-CTA kernel: 128 x 256 tiles.
// ---------------------------------------------------------------------------------------------
template <bool GROUPED>
__global__ void __launch_bounds__(kGemmThreads, 1)
    mx_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                   const GemmArgs a) {
    using L = typename std::conditional<GROUPED, Smem1Grouped, Smem1Dense>::type;
    constexpr int S = L::kStages;
    constexpr int kBBytes = kBN * kBK;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBar);
    uint64_t* empty = full + S;
    uint64_t* tmem_full = empty + S;        // [2]: accumulator g holds a finished tile
    uint64_t* acc_empty = tmem_full + 2;    // [2]: accumulator g has been read out
    uint64_t* ovl_free = acc_empty + 2;     // the epilogue has read the shared accumulator columns
    uint64_t* drain = ovl_free + 1;
    uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* abort = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
    int32_t* off = reinterpret_cast<int32_t*>(smem + L::kGroups);
    int32_t* pm = off + (kMaxGroups + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int g = 0; g < 2; ++g) {
            mbar_init(&tmem_full[g], 1);
            mbar_init(&acc_empty[g], kEpiWarps / 2);
        }
        mbar_init(ovl_free, kEpiWarps / 2);
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
    int tiles;
    if constexpr (GROUPED)
        tiles = setup_groups(a, off, pm, nullptr, a.tiles_n);
    else
        tiles = a.tiles_m * a.tiles_n;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_base_slot;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        int stage = 0;
        uint32_t phase = 0;
        int issued = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
            const Tile T = decode_tile1<GROUPED>(t, a, off, pm);
            const bool sfb1 = T.n0 + 128 < a.N;
            const uint32_t bytes = kBM * kBK + kBBytes + kSfaBytes + (sfb1 ? 1024u : 512u);
            for (int kb = 0; kb < a.nkb; ++kb) {
                if (!mbar_wait(&empty[stage], phase ^ 1u, abort, a.err, a.timeout_ns)) { ok = false; break; }
                __syncwarp();
                mbar_arrive_expect_tx_elect(&full[stage], bytes);
                tma_load_2d_elect(smem + L::kA + stage * kBM * kBK, &tmap_a, &full[stage], kb * kBK, T.a_row0);
                tma_load_2d_elect(smem + L::kB + stage * kBBytes, &tmap_b, &full[stage], kb * kBK, T.b_row0);
                bulk_load_elect(smem + L::kSfa + stage * kSfaBytes,
                                a.sfa + (static_cast<int64_t>(T.sfa_tile) * a.nkb + kb) * 512, 512, &full[stage]);
                bulk_load_elect(smem + L::kSfb + stage * kSfbBytes,
                                a.sfb + (static_cast<int64_t>(T.sfb_tile0) * a.nkb + kb) * 512, 512, &full[stage]);
                if (sfb1)
                    bulk_load_elect(smem + L::kSfb + stage * kSfbBytes + 512,
                                    a.sfb + (static_cast<int64_t>(T.sfb_tile1) * a.nkb + kb) * 512, 512, &full[stage]);
                ++issued;
                if (++stage == S) { stage = 0; phase ^= 1u; }
            }
        }
        if (!ok) {
            // Wait for the copies still in flight (the last min(issued, S) fills).
            int s = stage;
            uint32_t p = phase;
            for (int i = 0; i < min(issued, S); ++i) {
                if (--s < 0) { s = S - 1; p ^= 1u; }
                mbar_wait_drain(&full[s], p, a.timeout_ns);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        int stage = 0;
        uint32_t phase = 0, ovl_phase = 0, empty_phase = 0;
        bool ok = true;
        const uint32_t sfa_t = tmem_base + kSfCol;
        const uint32_t sfb_t = sfa_t + 4;
        int j = 0;
        for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++j) {
            if (j > 1) {                    // the accumulator's previous tile has been read out
                if (!mbar_wait(&acc_empty[j & 1], (empty_phase >> (j & 1)) & 1u, abort, a.err, a.timeout_ns)) {
                    ok = false;
                    break;
                }
                empty_phase ^= 1u << (j & 1);
            }
            if (j > 0) {                    // the previous tile's shared columns have been read
                if (!mbar_wait(ovl_free, ovl_phase, abort, a.err, a.timeout_ns)) { ok = false; break; }
                ovl_phase ^= 1u;
            }
            tc_fence_after();
            const uint32_t acc = tmem_base + ((j & 1) ? kAcc1Col : 0u);
            for (int kb = 0; kb < a.nkb; ++kb) {
                if (!mbar_wait(&full[stage], phase, abort, a.err, a.timeout_ns)) { ok = false; break; }
                __syncwarp();
                tc_fence_after();
                tc_cp_elect(sfa_t, sdesc_scale_block(smem_u32(smem + L::kSfa + stage * kSfaBytes)));
                tc_cp_elect(sfb_t, sdesc_scale_block(smem_u32(smem + L::kSfb + stage * kSfbBytes)));
                tc_cp_elect(sfb_t + 4, sdesc_scale_block(smem_u32(smem + L::kSfb + stage * kSfbBytes + 512)));
                const uint64_t adesc = sdesc_kmajor_sw128(smem_u32(smem + L::kA + stage * kBM * kBK));
                const uint64_t bdesc = sdesc_kmajor_sw128(smem_u32(smem + L::kB + stage * kBBytes));
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    // K-step k: +32 bytes inside the 128-byte swizzled rows; scale byte k.
                    tc_mma_mxf8_elect(acc, adesc + 2u * k, bdesc + 2u * k, idesc_mxf8_e4m3(kBM, kBN, k),
                                      sfa_t | (static_cast<uint32_t>(k) << 30), sfb_t | (static_cast<uint32_t>(k) << 30),
                                      (kb | k) != 0 ? 1u : 0u);
                }
                tc_commit_elect(&empty[stage]);
                if (++stage == S) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
            tc_commit_elect(&tmem_full[j & 1]);
        }
        // Every MMA issued by this warp has completed once `drain` fires.
        __syncwarp();
        tc_commit_elect(drain);
        mbar_wait_drain(drain, 0, a.timeout_ns);
    } else {
        // ---------------- epilogue ----------------
        const int q = warp & 3;             // TMEM lane quadrant this warp may access
        const int g = (warp - 2) >> 2;      // group: drains accumulator g, i.e. every other tile
        uint8_t* stage = smem + L::kStage + (warp - 2) * kStageBytes;
        const uint32_t ovl_addr = smem_u32(ovl_free);
        const uint32_t empty_addr = smem_u32(&acc_empty[g]);
        uint32_t full_phase = 0;
        for (int t = blockIdx.x + g * gridDim.x; t < tiles; t += 2 * gridDim.x) {
            const Tile T = decode_tile1<GROUPED>(t, a, off, pm);
            if (!mbar_wait(&tmem_full[g], full_phase, abort, a.err, a.timeout_ns)) break;
            full_phase ^= 1u;
            tc_fence_after();
            epilogue_tile<GROUPED>(a, T, tmem_base, g != 0, stage, ovl_addr, empty_addr, q, lane);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ---------------------------------------------------------------------------------------------
// CTA-pair kernel: 256 x 256 tiles, cluster of 2 (launched with cluster dimension 2).
// ---------------------------------------------------------------------------------------------
constexpr uint32_t kPairStageBytes = kBM * kBK + (kBN / 2) * kBK + kSfaBytes + kSfbBytes;   // per CTA

// EPI 0: C written as fp32 / BF16; EPI 1 (grouped only): the fused SwiGLU + MXFP8 epilogue.
template <bool GROUPED, int EPI = 0>
__global__ void __launch_bounds__(kGemmThreads, 1)
    mx_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                        const __grid_constant__ CUtensorMap tmap_sfa, const __grid_constant__ CUtensorMap tmap_sfb,
                        const GemmArgs a) {
    using L = typename std::conditional<GROUPED, SmemPairGrouped, SmemPairDense>::type;
    constexpr int S = L::kStages;
    constexpr int kBRows = kBN / 2;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBar);   // used in the leader CTA only
    uint64_t* empty = full + S;
    uint64_t* tmem_full = empty + S;        // [2]: accumulator g holds a finished tile (both CTAs)
    uint64_t* acc_empty = tmem_full + 2;    // [2], leader only: accumulator g read out in both CTAs
    uint64_t* ovl_free = acc_empty + 2;     // leader only: both CTAs' epilogues read the shared columns
    uint64_t* drain = ovl_free + 1;
    uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* abort = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
    uint32_t* issued_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc + 8);   // this CTA's operand fills
    int32_t* off = reinterpret_cast<int32_t*>(smem + L::kGroups);
    int32_t* pm128 = off + (kMaxGroups + 1);
    int32_t* pm256 = pm128 + (kMaxGroups + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int rank = static_cast<int>(cluster_ctarank());
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int g = 0; g < 2; ++g) {
            mbar_init(&tmem_full[g], 1);
            mbar_init(&acc_empty[g], kEpiWarps);    // one arrive per warp of one group in both CTAs
        }
        mbar_init(ovl_free, kEpiWarps);
        mbar_init(drain, 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmap_a);
        prefetch_tensormap(&tmap_b);
        prefetch_tensormap(&tmap_sfa);
        prefetch_tensormap(&tmap_sfb);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_base_slot, kTmemCols);
        tmem_relinquish_pair();
    }
    int tiles;
    if constexpr (GROUPED)
        tiles = setup_groups(a, off, pm128, pm256, a.tiles_n);
    else
        tiles = a.tiles_m * a.tiles_n;
    tc_fence_before();
    __syncthreads();
    cluster_sync();                         // both CTAs' barriers initialized before any remote signal
    tc_fence_after();
    const uint32_t tmem_base = *tmem_base_slot;

    if (warp == 0) {
        // ---------------- TMA producer (both CTAs; completions counted in the leader) ----------------
        int stage = 0;
        uint32_t phase = 0;
        int issued = 0;
        bool ok = true;
        for (int t = pair; t < tiles && ok; t += npairs) {
            const Tile T = decode_tile_pair<GROUPED>(t, rank, a, off, pm128, pm256);
            for (int kb = 0; kb < a.nkb; ++kb) {
                if (!mbar_wait(&empty[stage], phase ^ 1u, abort, a.err, a.timeout_ns)) { ok = false; break; }
                __syncwarp();
                const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
                if (leader) mbar_arrive_expect_tx_elect(&full[stage], 2 * kPairStageBytes);
                tma_load_2d_pair_elect(smem + L::kA + stage * kBM * kBK, &tmap_a, fb, kb * kBK, T.a_row0);
                tma_load_2d_pair_elect(smem + L::kB + stage * kBRows * kBK, &tmap_b, fb, kb * kBK, T.b_row0);
                // Scale blocks: the layout viewed as rows of 256 bytes, one block = 2 rows.
                tma_load_2d_pair_elect(smem + L::kSfa + stage * kSfaBytes, &tmap_sfa, fb, 0,
                                       2 * (T.sfa_tile * a.nkb + kb));
                tma_load_2d_pair_elect(smem + L::kSfb + stage * kSfbBytes, &tmap_sfb, fb, 0,
                                       2 * (T.sfb_tile0 * a.nkb + kb));
                tma_load_2d_pair_elect(smem + L::kSfb + stage * kSfbBytes + 512, &tmap_sfb, fb, 0,
                                       2 * (T.sfb_tile1 * a.nkb + kb));
                ++issued;
                if (++stage == S) { stage = 0; phase ^= 1u; }
            }
        }
        if (lane == 0) *issued_slot = static_cast<uint32_t>(issued);   // read by the leader's drain
    } else if (warp == 1) {
        if (leader) {
            // ---------------- MMA issuer (leader CTA, for both) ----------------
            int stage = 0;
            uint32_t phase = 0, ovl_phase = 0, empty_phase = 0;
            bool ok = true;
            const uint32_t sfa_t = tmem_base + kSfCol;
            const uint32_t sfb_t = sfa_t + 4;
            int j = 0;
            for (int t = pair; t < tiles && ok; t += npairs, ++j) {
                if (j > 1) {                // the accumulator's previous tile has been read out
                    if (!mbar_wait(&acc_empty[j & 1], (empty_phase >> (j & 1)) & 1u, abort, a.err,
                                   a.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    empty_phase ^= 1u << (j & 1);
                }
                if (j > 0) {                // the previous tile's shared columns have been read
                    if (!mbar_wait(ovl_free, ovl_phase, abort, a.err, a.timeout_ns)) { ok = false; break; }
                    ovl_phase ^= 1u;
                }
                tc_fence_after();
                const uint32_t acc = tmem_base + ((j & 1) ? kAcc1Col : 0u);
                for (int kb = 0; kb < a.nkb; ++kb) {
                    if (!mbar_wait(&full[stage], phase, abort, a.err, a.timeout_ns)) { ok = false; break; }
                    __syncwarp();
                    tc_fence_after();
                    tc_cp_pair_elect(sfa_t, sdesc_scale_block(smem_u32(smem + L::kSfa + stage * kSfaBytes)));
                    tc_cp_pair_elect(sfb_t, sdesc_scale_block(smem_u32(smem + L::kSfb + stage * kSfbBytes)));
                    tc_cp_pair_elect(sfb_t + 4, sdesc_scale_block(smem_u32(smem + L::kSfb + stage * kSfbBytes + 512)));
                    const uint64_t adesc = sdesc_kmajor_sw128(smem_u32(smem + L::kA + stage * kBM * kBK));
                    const uint64_t bdesc = sdesc_kmajor_sw128(smem_u32(smem + L::kB + stage * kBRows * kBK));
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        tc_mma_mxf8_pair_elect(acc, adesc + 2u * k, bdesc + 2u * k, idesc_mxf8_e4m3(2 * kBM, kBN, k),
                                               sfa_t | (static_cast<uint32_t>(k) << 30),
                                               sfb_t | (static_cast<uint32_t>(k) << 30), (kb | k) != 0 ? 1u : 0u);
                    }
                    tc_commit_pair_elect(&empty[stage], 0x3);     // both CTAs' stage is free again
                    if (++stage == S) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                tc_commit_pair_elect(&tmem_full[j & 1], 0x3);
            }
            __syncwarp();
            tc_commit_pair_elect(drain, 0x1);
            mbar_wait_drain(drain, 0, a.timeout_ns);
        }
    } else {
        // ---------------- epilogue (both CTAs) ----------------
        const int q = warp & 3;             // TMEM lane quadrant this warp may access
        const int g = (warp - 2) >> 2;      // group: drains accumulator g, i.e. every other tile
        uint8_t* stage = smem + L::kStage + (warp - 2) * kStageBytes;
        const uint32_t ovl_addr = mapa_shared(smem_u32(ovl_free), 0);
        const uint32_t empty_addr = mapa_shared(smem_u32(&acc_empty[g]), 0);
        uint32_t full_phase = 0;
        for (int t = pair + g * npairs; t < tiles; t += 2 * npairs) {
            const Tile T = decode_tile_pair<GROUPED>(t, rank, a, off, pm128, pm256);
            if (!mbar_wait(&tmem_full[g], full_phase, abort, a.err, a.timeout_ns)) break;
            full_phase ^= 1u;
            tc_fence_after();
            if constexpr (EPI == 0)
                epilogue_tile<GROUPED>(a, T, tmem_base, g != 0, stage, ovl_addr, empty_addr, q, lane);
            else
                epilogue_swiglu_tile(a, T, tmem_base, g != 0, ovl_addr, empty_addr, q, lane);
        }
    }

    // Neither CTA leaves (or frees TMEM) while the pair still has MMAs, copies or signals in flight.
    // Past the first cluster barrier no role of either CTA issues anything. Both CTAs' operand
    // copies complete on the leader's `full` barriers; after an expired wait the two producers may
    // have stopped at different fills, so the leader drains the last S fills either CTA issued:
    // for a fill only one CTA issued it supplies the missing half of the stage's transaction count
    // (the bytes that were never requested, or its own arrival for the peer's bytes) and waits for
    // the copies that were. On the normal path every phase has completed and these waits return
    // at once.
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (leader && warp == 0 && lane == 0) {
        const uint32_t mine = *issued_slot;
        const uint32_t peer = ld_shared_cluster_u32(mapa_shared(smem_u32(issued_slot), 1));
        const uint32_t hi = max(mine, peer);
        for (uint32_t i = hi > static_cast<uint32_t>(S) ? hi - S : 0u; i < hi; ++i) {
            uint64_t* bar = &full[i % S];
            if (i >= mine)
                mbar_arrive_expect_tx(bar, kPairStageBytes);    // the peer's copies only
            else if (i >= peer)
                mbar_complete_tx(bar, kPairStageBytes);         // the peer never requested its half
            mbar_wait_drain(bar, (i / S) & 1u, a.timeout_ns);
        }
    }
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

}  // namespace mx
