// MXFP8 quantizer: rowwise and/or columnwise, optionally writing the tensor-core scale layout
// directly, over one tensor or a list of tensors in one launch.
//
// The paper ("End-to-End MXFP8 Reinforcement Learning on Blackwell", Figure 1 and Table 6) has the
// learner quantize BF16 masters and activations and then rearrange the E8M0 scales ("scale
// rearrangement", 2.6 ms per micro-batch, more than the 2.2 ms of quantization). Here both happen in
// one HBM pass: a CTA iteration owns a 128 x 128 BF16 tile, whose rowwise scales (128 rows x 4
// K-blocks) and columnwise scales (128 K-rows x 4 M-blocks) are each exactly one 512-byte block of
// the tensor-core scale layout, so the swizzled scales leave the CTA as one coalesced 512-byte store.
// At weight synchronization every weight of the model is quantized (Figure 1); the multi-tensor
// form walks the tiles of all of them as one tile space, so one persistent launch covers the model.
//
// Rule (OCP MX v1.0; the paper's "E8M0 scales keep only the exponent", Table 10 F6): per 32-block,
// e = floor(log2 amax) - 8 clamped to [-127, 127], scale byte e + 127; elements RNE(x * 2^-e)
// saturated to +-448 in E4M3. For BF16 input floor(log2 amax) is the biased exponent field minus
// 127, so the scale byte is max(E_amax - 8, 0), computed on integer bits. x * 2^-e is exact in fp32
// (a packed fp32x2 multiply) and one cvt.rn.satfinite rounds it. Blocks holding NaN or Inf get
// scale 0xFF and element bytes sign|0x7F.
//
// This file must not be compiled with flush-to-zero: BF16 subnormal inputs scaled by 2^127 are
// normal E4M3 values.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace mx {

constexpr int kQTile = 128;          // rows and columns of a quantizer tile
constexpr int kQThreads = 256;
constexpr int kQMaxTensors = 192;    // tensors per multi-tensor launch (kernel parameters < 32 KB)

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// max(|a|, |b|) per BF16 half, NaN-propagating (a NaN operand gives the canonical NaN 0x7FFF);
// the sign bits of the result are garbage and are masked by the caller.
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Scale byte from the largest BF16 magnitude bits of a block (0 .. 0x7FFF).
__device__ __forceinline__ uint32_t scale_byte_from_amax(uint32_t amax_bits) {
    if (amax_bits >= 0x7F80u) return 0xFFu;            // Inf or NaN in the block
    const int E = static_cast<int>(amax_bits >> 7);    // biased exponent of amax (0 for subnormal/zero)
    return static_cast<uint32_t>(E > 8 ? E - 8 : 0);
}

// {2^-e, 2^-e} as a packed fp32 pair for scale byte s = e + 127 <= 246: biased exponent 254 - s.
__device__ __forceinline__ uint64_t inv_scale2(uint32_t s) {
    const uint32_t f = (254u - s) << 23;
    return (static_cast<uint64_t>(f) << 32) | f;
}

// E4M3 codes of four values given as fp32 bit patterns (e0 -> bits 0-7 ... e3 -> bits 24-31),
// after scaling all by the packed pair inv2.
__device__ __forceinline__ uint32_t enc_quad(uint32_t e0, uint32_t e1, uint32_t e2, uint32_t e3, uint64_t inv2) {
    uint32_t r;
    asm("{\n\t.reg .b64 x0, x1, y0, y1;\n\t.reg .b32 l0, h0, l1, h1;\n\t.reg .b16 c0, c1;\n\t"
        "mov.b64 x0, {%1, %2};\n\t"
        "mov.b64 x1, {%3, %4};\n\t"
        "mul.rn.f32x2 y0, x0, %5;\n\t"
        "mul.rn.f32x2 y1, x1, %5;\n\t"
        "mov.b64 {l0, h0}, y0;\n\t"
        "mov.b64 {l1, h1}, y1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 c0, h0, l0;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 c1, h1, l1;\n\t"
        "mov.b32 %0, {c0, c1};\n\t}"
        : "=r"(r)
        : "r"(e0), "r"(e1), "r"(e2), "r"(e3), "l"(inv2));
    return r;
}

// Four BF16 (two words, element 0 in the low half of w0) -> four E4M3 bytes (element 0 in bits
// 0-7), scaled by the packed pair inv2.
__device__ __forceinline__ uint32_t enc_words(uint32_t w0, uint32_t w1, uint64_t inv2) {
    uint32_t r;
    asm("{\n\t.reg .b64 x0, x1, y0, y1;\n\t.reg .b32 l0, h0, l1, h1;\n\t.reg .b16 c0, c1;\n\t"
        "shl.b32 l0, %1, 16;\n\t"
        "and.b32 h0, %1, 0xFFFF0000;\n\t"
        "shl.b32 l1, %2, 16;\n\t"
        "and.b32 h1, %2, 0xFFFF0000;\n\t"
        "mov.b64 x0, {l0, h0};\n\t"
        "mov.b64 x1, {l1, h1};\n\t"
        "mul.rn.f32x2 y0, x0, %3;\n\t"
        "mul.rn.f32x2 y1, x1, %3;\n\t"
        "mov.b64 {l0, h0}, y0;\n\t"
        "mov.b64 {l1, h1}, y1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 c0, h0, l0;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 c1, h1, l1;\n\t"
        "mov.b32 %0, {c0, c1};\n\t}"
        : "=r"(r)
        : "r"(w0), "r"(w1), "l"(inv2));
    return r;
}

// Eight BF16 (one 16-byte chunk, element 0 in the low half of v.x) -> eight E4M3 bytes.
__device__ __forceinline__ uint2 encode_chunk(const uint4 v, uint32_t s) {
    uint2 o;
    if (s != 0xFFu) {
        const uint64_t inv2 = inv_scale2(s);
        o.x = enc_words(v.x, v.y, inv2);
        o.y = enc_words(v.z, v.w, inv2);
    } else {
        // NaN/Inf block: every element byte is sign | 0x7F.
        const uint32_t m = 0x7F7F7F7Fu;
        o.x = m | ((v.x >> 8) & 0x80u) | ((v.x >> 16) & 0x8000u) | ((v.y << 8) & 0x800000u) | (v.y & 0x80000000u);
        o.y = m | ((v.z >> 8) & 0x80u) | ((v.z >> 16) & 0x8000u) | ((v.w << 8) & 0x800000u) | (v.w & 0x80000000u);
    }
    return o;
}

struct QTensor {
    const uint16_t* x;
    uint8_t* q_row;
    uint8_t* s_row;
    uint8_t* q_col;
    uint8_t* s_col;
    int64_t M, K, ldx;
    int64_t tile_start;       // first tile of this tensor in the launch's tile space
    int32_t tiles_m, tiles_k;
    int32_t vec32;            // x rows and q_row 32-byte aligned: 256-bit loads and stores
    int32_t col_vec32;        // q_col 32-byte aligned: 256-bit stores of the transposed copy
    // Fused comparison (mx_quantize_compare_multi): the grid the codes and swizzled scales are
    // compared with, and the result slots 2 res (codes) and 2 res + 1 (scales).
    const uint8_t* ref_q;
    const uint8_t* ref_s;
    int32_t res;
    int32_t ref_vec32;        // ref_q 32-byte aligned: 256-bit loads
};

struct Block32 {
    uint4 v[4];               // 32 BF16, element 0 in the low half of v[0].x
};

__device__ __forceinline__ void ld_stream_v8(const void* p, uint4& a, uint4& b) {
    asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
                 : "l"(p));
}

__device__ __forceinline__ uint4 ld_cached_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ void st_v8(void* p, const uint4& a, const uint4& b) {
    asm volatile("st.global.v8.u32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a.x), "r"(a.y),
                 "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
                 : "memory");
}

template <int NT>
struct QuantArgs {
    int n;                    // tensors in this launch
    int swz;                  // write the tensor-core scale layout (else raw scales)
    int64_t total_tiles;
    unsigned long long* cmp_counts;   // fused comparison: differing bytes per result slot
    long long* cmp_firsts;            // ... and the index of the first (-1 if none)
    QTensor t[NT];
};

// Nonzero bytes of x -> 0x01 in that byte.
__device__ __forceinline__ uint32_t differing_bytes(uint32_t x) {
    x |= x >> 4;
    x |= x >> 2;
    x |= x >> 1;
    return x & 0x01010101u;
}

// Adds the differing bytes of `mine` against `ref` (16 bytes at buffer offset `base`) to cnt and
// lowers first to the smallest differing offset.
__device__ __forceinline__ void compare16(const uint4& mine, const uint4& ref, int64_t base, unsigned long long& cnt,
                                          unsigned long long& first) {
    const uint32_t d[4] = {differing_bytes(mine.x ^ ref.x), differing_bytes(mine.y ^ ref.y),
                           differing_bytes(mine.z ^ ref.z), differing_bytes(mine.w ^ ref.w)};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        if (d[k]) {
            cnt += __popc(d[k]);
            const unsigned long long idx = static_cast<unsigned long long>(base + 4 * k + (__ffs(d[k]) - 1) / 8);
            first = idx < first ? idx : first;
        }
    }
}

// Adds one warp's counts to result slot `slot` (only when some lane saw a difference).
__device__ __forceinline__ void flush_compare(unsigned long long cnt, unsigned long long first,
                                              unsigned long long* counts, long long* firsts, int slot) {
    if (__any_sync(0xFFFFFFFFu, cnt != 0)) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            cnt += __shfl_xor_sync(0xFFFFFFFFu, cnt, o);
            const unsigned long long f = __shfl_xor_sync(0xFFFFFFFFu, first, o);
            first = f < first ? f : first;
        }
        if ((threadIdx.x & 31) == 0) {
            atomicAdd(&counts[slot], cnt);
            atomicMin(reinterpret_cast<unsigned long long*>(&firsts[slot]), first);
        }
    }
}

struct TileRef {
    int i;                    // tensor index
    int64_t m0, k0;
    int mt, kt;
    bool full;                // the whole 128 x 128 tile lies inside the tensor
};

template <int NT>
__device__ __forceinline__ TileRef decode_qtile(const QuantArgs<NT>& a, int64_t t) {
    int i = 0;
    if constexpr (NT > 1) {
        int lo = 0, hi = a.n - 1;    // largest i with tile_start <= t
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (a.t[mid].tile_start <= t) lo = mid; else hi = mid - 1;
        }
        i = lo;
    }
    const QTensor& T = a.t[i];
    const int64_t local = t - T.tile_start;
    TileRef r;
    r.i = i;
    r.mt = static_cast<int>(local / T.tiles_k);
    r.kt = static_cast<int>(local % T.tiles_k);
    r.m0 = static_cast<int64_t>(r.mt) * kQTile;
    r.k0 = static_cast<int64_t>(r.kt) * kQTile;
    r.full = (r.m0 + kQTile <= T.M) && (r.k0 + kQTile <= T.K);
    return r;
}

// ---- rowwise-only kernel: one thread per 32-element block ----------------------------------
//
// Thread tid owns blocks (row tid >> 2, K-block tid & 3) and (row 64 + (tid >> 2), same K-block) of
// the 128 x 128 tile: the block's amax, scale and 32 codes need no cross-lane exchange, and its 64
// input bytes and 32 output bytes move with 256-bit accesses when the tensor is 32-byte aligned.

__device__ __forceinline__ void load_block(const QTensor& T, int64_t row, int64_t col, bool ok, Block32& b) {
    if (!ok) {
        b.v[0] = b.v[1] = b.v[2] = b.v[3] = make_uint4(0, 0, 0, 0);
        return;
    }
    const uint16_t* p = T.x + row * T.ldx + col;
    if (T.vec32) {
        ld_stream_v8(p, b.v[0], b.v[1]);
        ld_stream_v8(p + 16, b.v[2], b.v[3]);
    } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) b.v[j] = ld_cached_v4(p + 8 * j);
    }
}

template <int NT>
__device__ __forceinline__ void load_row_tile(const QuantArgs<NT>& a, const TileRef& r, Block32 (&b)[2], int tid) {
    const QTensor& T = a.t[r.i];
    const int64_t col = r.k0 + (tid & 3) * 32;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int64_t row = r.m0 + h * 64 + (tid >> 2);
        load_block(T, row, col, r.full || (row < T.M && col < T.K), b[h]);
    }
}

// SPLIT == false: the whole next tile is loaded into a second register set at the top of each
// iteration. SPLIT == true: each half of the next tile is loaded into the registers of the same half
// of the current tile as soon as that half is encoded (no second set; loads issued later). The host
// picks SPLIT for long per-CTA tile walks, where it measured faster, and the other form for short ones.
// CMP == true (weight synchronization, Table 11's byte comparison fused into the quantizer): the
// codes and the swizzled scale block each tile writes are also compared with a reference grid (the
// sampler's copy), read once; differing bytes and the first differing offset go to the tensor's
// result slots, as mx_grid_equal would report them for the written grid.
template <int NT, bool SPLIT, bool CMP = false>
__global__ void __launch_bounds__(kQThreads, 2) quantize_rowwise_kernel(const __grid_constant__ QuantArgs<NT> a) {
    __shared__ __align__(16) uint8_t atom[512];
    const int tid = threadIdx.x;

    const int64_t per = (a.total_tiles + gridDim.x - 1) / gridDim.x;
    const int64_t t_begin = static_cast<int64_t>(blockIdx.x) * per;
    const int64_t t_end = min(a.total_tiles, t_begin + per);
    Block32 cur[2], nxt[SPLIT ? 1 : 2];
    uint4 ref[2][2];                                     // CMP: the reference codes of this thread's blocks
    TileRef rc, rn;
    // CMP: reference codes of block h of tile r, loaded one tile ahead like the BF16 input.
    auto load_ref = [&](const TileRef& r, int h) {
        const QTensor& Tr = a.t[r.i];
        const int64_t row = r.m0 + h * 64 + (tid >> 2);
        const int64_t col = r.k0 + (tid & 3) * 32;
        if (r.full || (row < Tr.M && col < Tr.K)) {
            const uint8_t* rq = Tr.ref_q + row * Tr.K + col;
            if (Tr.ref_vec32) {
                ld_stream_v8(rq, ref[h][0], ref[h][1]);
            } else {
                ref[h][0] = ld_cached_v4(rq);
                ref[h][1] = ld_cached_v4(rq + 16);
            }
        }
    };
    if (t_begin < t_end) {
        rc = decode_qtile(a, t_begin);
        load_row_tile(a, rc, cur, tid);
        if constexpr (CMP) {
            load_ref(rc, 0);
            load_ref(rc, 1);
        }
    }
    for (int64_t t = t_begin; t < t_end; ++t) {
        if (t + 1 < t_end) {
            rn = rc;
            if (++rn.kt == a.t[rn.i].tiles_k) {
                rn.kt = 0;
                if (++rn.mt == a.t[rn.i].tiles_m) {
                    rn.mt = 0;
                    ++rn.i;
                }
            }
            const QTensor& Tn = a.t[rn.i];
            rn.m0 = static_cast<int64_t>(rn.mt) * kQTile;
            rn.k0 = static_cast<int64_t>(rn.kt) * kQTile;
            rn.full = (rn.m0 + kQTile <= Tn.M) && (rn.k0 + kQTile <= Tn.K);
            if constexpr (!SPLIT) load_row_tile(a, rn, nxt, tid);
        }
        const QTensor& T = a.t[rc.i];
        const int kb = tid & 3;
        const int64_t col = rc.k0 + kb * 32;
        unsigned long long ecnt = 0, efirst = ~0ull;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int r = h * 64 + (tid >> 2);           // row inside the tile
            const int64_t row = rc.m0 + r;
            const bool valid = rc.full || (row < T.M && col < T.K);
            const Block32& b = cur[h];
            uint32_t m = bf16x2_absmax(bf16x2_absmax(b.v[0].x, b.v[0].y), bf16x2_absmax(b.v[0].z, b.v[0].w));
#pragma unroll
            for (int j = 1; j < 4; ++j)
                m = bf16x2_absmax(m, bf16x2_absmax(bf16x2_absmax(b.v[j].x, b.v[j].y), bf16x2_absmax(b.v[j].z, b.v[j].w)));
            m &= 0x7FFF7FFFu;
            const uint32_t s = scale_byte_from_amax(max(m & 0xFFFFu, m >> 16));
            uint4 o0, o1;
            uint2 e;
            e = encode_chunk(b.v[0], s);
            o0.x = e.x; o0.y = e.y;
            e = encode_chunk(b.v[1], s);
            o0.z = e.x; o0.w = e.y;
            e = encode_chunk(b.v[2], s);
            o1.x = e.x; o1.y = e.y;
            e = encode_chunk(b.v[3], s);
            o1.z = e.x; o1.w = e.y;
            if (valid) {
                uint8_t* q = T.q_row + row * T.K + col;
                if (T.vec32) {
                    st_v8(q, o0, o1);
                } else {
                    reinterpret_cast<uint4*>(q)[0] = o0;
                    reinterpret_cast<uint4*>(q)[1] = o1;
                }
                if constexpr (CMP) {
                    compare16(o0, ref[h][0], row * T.K + col, ecnt, efirst);
                    compare16(o1, ref[h][1], row * T.K + col + 16, ecnt, efirst);
                }
            }
            atom[(r & 31) * 16 + (r >> 5) * 4 + kb] = valid ? static_cast<uint8_t>(s) : 0;
            if (SPLIT && t + 1 < t_end) {
                const QTensor& Tn = a.t[rn.i];
                const int64_t rown = rn.m0 + h * 64 + (tid >> 2);
                const int64_t coln = rn.k0 + kb * 32;
                load_block(Tn, rown, coln, rn.full || (rown < Tn.M && coln < Tn.K), cur[h]);
            }
            if (CMP && t + 1 < t_end) load_ref(rn, h);
        }
        if constexpr (CMP) flush_compare(ecnt, efirst, a.cmp_counts, a.cmp_firsts, 2 * T.res);
        __syncthreads();
        if (a.swz) {
            if (tid < 32) {
                const int64_t soff = (static_cast<int64_t>(rc.mt) * T.tiles_k + rc.kt) * 512;
                const uint4 mine = reinterpret_cast<const uint4*>(atom)[tid];
                reinterpret_cast<uint4*>(T.s_row + soff)[tid] = mine;
                if constexpr (CMP) {
                    unsigned long long scnt = 0, sfirst = ~0ull;
                    compare16(mine, ld_cached_v4(T.ref_s + soff + tid * 16), soff + tid * 16, scnt, sfirst);
                    flush_compare(scnt, sfirst, a.cmp_counts, a.cmp_firsts, 2 * T.res + 1);
                }
            }
        } else if (tid < kQTile) {
            const int64_t kblocks = T.K / 32;
            const int64_t m = rc.m0 + tid;
            const int64_t nb = (kblocks - rc.kt * 4 < 4 ? kblocks - rc.kt * 4 : 4);
            if (m < T.M)
                for (int q = 0; q < nb; ++q)
                    T.s_row[m * kblocks + rc.kt * 4 + q] = atom[(tid & 31) * 16 + (tid >> 5) * 4 + q];
        }
        __syncthreads();
        if constexpr (!SPLIT) {
            cur[0] = nxt[0];
            cur[1] = nxt[1];
        }
        rc = rn;
    }
}

// ---- rowwise + columnwise kernel -------------------------------------------------------------
//
// Same tile walk and block-per-thread rowwise pass as above. Each thread also stages its two
// BF16 blocks in shared memory (128 rows x 256 bytes; 16-byte chunks XOR-swizzled so that both
// these row-block writes and the column reads below are free of bank conflicts). Then thread t
// quantizes tile columns 2 (t & 63) and 2 (t & 63) + 1 over the 32-row M-block t >> 6: each 32-bit
// shared word holds one row's pair of those columns, so one pass of packed BF16 maxima gives both
// columns' amax. Its 2 x 32 codes are two 32-byte pieces of the transposed copy ([K, M]).

// Byte offset of 16-byte chunk c (0..15) of row r in the shared tile.
__device__ __forceinline__ uint32_t qtile_chunk(int r, int c) {
    return static_cast<uint32_t>(r * 256 + ((c ^ (((c >> 3) & 1) << 1) ^ (r & 1)) << 4));
}

__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t saddr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(saddr));
    return v;
}

// Largest magnitude bits of each half over w[0..31] (two columns of a 32-row block), as a tree of
// depth 5 rather than a chain of 32 dependent maxima.
__device__ __forceinline__ uint32_t col_pair_absmax(const uint32_t (&w)[32]) {
    uint32_t m[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) m[i] = bf16x2_absmax(w[2 * i], w[2 * i + 1]);
#pragma unroll
    for (int n = 8; n >= 1; n >>= 1)
#pragma unroll
        for (int i = 0; i < n; ++i) m[i] = bf16x2_absmax(m[i], m[i + n]);
    return m[0] & 0x7FFF7FFFu;
}

// The 32 BF16 of one column (the low or the high halves of w[0..31]) -> 32 E4M3 bytes, row i in
// byte i of the result.
__device__ __forceinline__ void encode_col32(const uint32_t (&w)[32], uint32_t s, bool hi, uint32_t (&o)[8]) {
    if (s != 0xFFu) {
        const uint64_t inv2 = inv_scale2(s);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            uint32_t e[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) e[i] = hi ? (w[4 * q + i] & 0xFFFF0000u) : (w[4 * q + i] << 16);
            o[q] = enc_quad(e[0], e[1], e[2], e[3], inv2);
        }
    } else {
        // NaN/Inf block: every element byte is sign | 0x7F.
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            uint32_t r = 0x7F7F7F7Fu;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t sign = hi ? (w[4 * q + i] >> 31) : ((w[4 * q + i] >> 15) & 1u);
                r |= sign << (8 * i + 7);
            }
            o[q] = r;
        }
    }
}

template <bool ROW, int NT>
__global__ void __launch_bounds__(kQThreads, 2) quantize_rowcol_kernel(const __grid_constant__ QuantArgs<NT> a) {
    __shared__ __align__(128) uint8_t tile[kQTile * 256];
    __shared__ __align__(16) uint8_t atom_row[512];
    __shared__ __align__(16) uint8_t atom_col[512];
    const int tid = threadIdx.x;
    const uint32_t tile_s = smem_u32(tile);

    const int64_t per = (a.total_tiles + gridDim.x - 1) / gridDim.x;
    const int64_t t_begin = static_cast<int64_t>(blockIdx.x) * per;
    const int64_t t_end = min(a.total_tiles, t_begin + per);
    Block32 cur[2];
    TileRef rc, rn;
    if (t_begin < t_end) {
        rc = decode_qtile(a, t_begin);
        load_row_tile(a, rc, cur, tid);
    }
    for (int64_t t = t_begin; t < t_end; ++t) {
        if (t + 1 < t_end) {
            rn = rc;
            if (++rn.kt == a.t[rn.i].tiles_k) {
                rn.kt = 0;
                if (++rn.mt == a.t[rn.i].tiles_m) {
                    rn.mt = 0;
                    ++rn.i;
                }
            }
            const QTensor& Tn = a.t[rn.i];
            rn.m0 = static_cast<int64_t>(rn.mt) * kQTile;
            rn.k0 = static_cast<int64_t>(rn.kt) * kQTile;
            rn.full = (rn.m0 + kQTile <= Tn.M) && (rn.k0 + kQTile <= Tn.K);
        }
        const QTensor& T = a.t[rc.i];
        const int kb = tid & 3;
        const int64_t col = rc.k0 + kb * 32;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int r = h * 64 + (tid >> 2);           // row inside the tile
            const Block32& b = cur[h];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                st_shared_v4(tile_s + qtile_chunk(r, kb * 4 + j), b.v[j].x, b.v[j].y, b.v[j].z, b.v[j].w);
            if constexpr (ROW) {
                const int64_t row = rc.m0 + r;
                const bool valid = rc.full || (row < T.M && col < T.K);
                uint32_t m = bf16x2_absmax(bf16x2_absmax(b.v[0].x, b.v[0].y), bf16x2_absmax(b.v[0].z, b.v[0].w));
#pragma unroll
                for (int j = 1; j < 4; ++j)
                    m = bf16x2_absmax(m, bf16x2_absmax(bf16x2_absmax(b.v[j].x, b.v[j].y),
                                                       bf16x2_absmax(b.v[j].z, b.v[j].w)));
                m &= 0x7FFF7FFFu;
                const uint32_t s = scale_byte_from_amax(max(m & 0xFFFFu, m >> 16));
                uint4 o0, o1;
                uint2 e;
                e = encode_chunk(b.v[0], s);
                o0.x = e.x; o0.y = e.y;
                e = encode_chunk(b.v[1], s);
                o0.z = e.x; o0.w = e.y;
                e = encode_chunk(b.v[2], s);
                o1.x = e.x; o1.y = e.y;
                e = encode_chunk(b.v[3], s);
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
                atom_row[(r & 31) * 16 + (r >> 5) * 4 + kb] = valid ? static_cast<uint8_t>(s) : 0;
            }
            // Half h of the tile is in shared memory and encoded: the next tile's half h loads into
            // the same registers and stays in flight through the rest of this tile.
            if (t + 1 < t_end) {
                const QTensor& Tn = a.t[rn.i];
                const int64_t rown = rn.m0 + h * 64 + (tid >> 2);
                const int64_t coln = rn.k0 + kb * 32;
                load_block(Tn, rown, coln, rn.full || (rown < Tn.M && coln < Tn.K), cur[h]);
            }
        }
        __syncthreads();
        {
            const int cp = tid & 63;                     // column pair: tile columns 2 cp, 2 cp + 1
            const int mb = tid >> 6;                     // 32-row M-block
            uint32_t w[32];
#pragma unroll
            for (int i = 0; i < 32; ++i)
                w[i] = ld_shared_u32(tile_s + qtile_chunk(mb * 32 + i, cp >> 2) + (cp & 3) * 4);
            const uint32_t m = col_pair_absmax(w);
            const int64_t kc = rc.k0 + 2 * cp;           // K-row of the transposed copy (low halves)
            const int64_t mr = rc.m0 + 32 * mb;
            const bool mok = rc.full || mr < T.M;        // M % 32 == 0: a block is all in or all out
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const uint32_t s = scale_byte_from_amax(hh ? (m >> 16) : (m & 0xFFFFu));
                const bool ok = mok && (rc.full || kc + hh < T.K);
                uint32_t o[8];
                encode_col32(w, s, hh != 0, o);
                if (ok) {
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
                atom_col[(kk & 31) * 16 + (kk >> 5) * 4 + mb] = ok ? static_cast<uint8_t>(s) : 0;
            }
        }
        __syncthreads();
        // Scale output: one 512-byte block of the tensor-core layout per direction, or raw bytes.
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
        {
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
        __syncthreads();
        rc = rn;
    }
}

}  // namespace mx
