/*
 * libmx -- MXFP8 quantize, scale layout, block-scaled GEMM and grid equality on NVIDIA B200
 * (sm_100a). C ABI: plain pointers and sizes; no allocation, no host synchronisation (except
 * mx_device_error), every call asynchronous on `stream`.
 *
 * The operations follow "End-to-End MXFP8 Reinforcement Learning on Blackwell: What Matching
 * Buys, When It Pays Off, and How It Fails" (W. Zhang, arXiv 2610.34915):
 *   - Figure 1: the learner computes with MXFP8 GEMMs over BF16 master weights; at every weight
 *     synchronization the weights are quantized with the learner's own quantizer, so the sampler
 *     receives the learner's grid, and the sampler re-derives its kernel layouts in place;
 *   - Table 6: per micro-batch the MXFP8 path spends time in "MXFP8 quantization", "scale
 *     rearrangement" and "GEMM";
 *   - Table 10 (F3, F4, F6) and Table 11 (byte comparison): the synchronized weight, scale and
 *     kernel layout must equal the learner's quantization byte for byte.
 * The pages do not print the quantization rule or the scale layout. The rule is the OCP MX v1.0
 * one for MXFP8, the layout NVIDIA's sm_100 block-scaling-factor layout:
 *   - elements: FP8 E4M3 ("fn": max 448, no infinities, S.1111.111 = NaN);
 *   - one E8M0 scale per 32 consecutive elements along K: e = floor(log2(amax)) - 8, clamped to
 *     [-127, 127], stored as e + 127; an all-zero block gets byte 0;
 *   - element = round-to-nearest-even(x * 2^-e), saturated to +-448, signed zero kept;
 *   - a block containing NaN or +-Inf gets scale 0xFF and every element byte sign | 0x7F;
 *   - tensor-core scale layout: pad a [R, C] scale matrix to R' = ceil(R/128)*128 rows and
 *     C' = ceil(C/4)*4 columns (pad bytes 0x00); 128 x 4 blocks of 512 bytes, row-block major;
 *     inside a block, scale (r, c) is at byte (r % 32) * 16 + ((r % 128) / 32) * 4 + c % 4.
 *
 * Memory: the caller allocates and owns every buffer. All buffers named "device" must be device
 * memory of the current CUDA device; all of them must be 16-byte aligned. Buffers must not
 * overlap unless stated.
 *
 * Errors: arguments are checked on the host before any launch and reported as mx_status; nothing
 * is launched when a check fails. MX_ERR_CUDA reports a failed launch or driver call. Device-side
 * faults that a kernel detects (a bounded wait that expired, invalid grouped-GEMM row offsets)
 * set bits in a device status word readable with mx_device_error.
 */
#ifndef MX_H
#define MX_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (cudaStream_t / CUstream); NULL is the legacy default stream. */
typedef struct CUstream_st* mx_stream;

typedef enum {
    MX_OK = 0,
    MX_ERR_ARG = -1,          /* null pointer, negative size, bad flag or enum value */
    MX_ERR_SHAPE = -2,        /* a size the operation cannot take (e.g. K % 32 != 0) */
    MX_ERR_ALIGN = -3,        /* pointer or leading dimension not 16-byte aligned */
    MX_ERR_CUDA = -4,         /* a CUDA launch or driver call failed */
    MX_ERR_UNSUPPORTED = -5,  /* device is not sm_100 / feature unavailable */
    MX_ERR_DEVICE = -6        /* mx_device_error found a device-side error bit set */
} mx_status;

/* mx_quantize flags. */
enum { MX_ROWWISE = 1, MX_COLWISE = 2, MX_SWIZZLE = 4 };

/* GEMM output element type. */
typedef enum { MX_OUT_F32 = 0, MX_OUT_BF16 = 1 } mx_out_dtype;

/* Bytes of the tensor-core scale layout for a [rows, kblocks] scale matrix:
 * ceil(rows/128)*128 * ceil(kblocks/4)*4. Returns -1 for negative sizes. */
int64_t mx_swizzled_scale_bytes(int64_t rows, int64_t kblocks);

/*
 * MXFP8 quantization of a BF16 matrix x[M, K] (device, row stride ld_x elements), the learner's
 * quantizer of Figure 1 and Table 6 ("MXFP8 quantization"), with the scale rearrangement of
 * Table 6 fused when MX_SWIZZLE is set. One pass over x produces any of:
 *   MX_ROWWISE: q_row[M, K] E4M3 codes (packed, row stride K) and s_row, the E8M0 scales of the
 *               32-blocks along K: raw [M, K/32] (packed), or with MX_SWIZZLE the tensor-core
 *               layout of that matrix (mx_swizzled_scale_bytes(M, K/32) bytes, pads written 0).
 *   MX_COLWISE: q_col[K, M] = the rowwise quantization of x^T (blocks of 32 along M, stored
 *               K-major for the transposed GEMM operands of dgrad / wgrad) and s_col: raw
 *               [K, M/32] or swizzled (mx_swizzled_scale_bytes(K, M/32) bytes).
 * Requirements: K % 32 == 0; M % 32 == 0 if MX_COLWISE; M, K < 2^31; ld_x >= K and ld_x % 8 == 0; at least
 * one of MX_ROWWISE / MX_COLWISE; the pointers of each requested direction non-NULL (others are
 * ignored); all pointers 16-byte aligned. M == 0 or K == 0 is a no-op.
 * Result is bit-exact to the rule in the header comment.
 */
mx_status mx_quantize(const void* x_bf16, int64_t M, int64_t K, int64_t ld_x, int flags,
                      uint8_t* q_row, uint8_t* s_row, uint8_t* q_col, uint8_t* s_col,
                      mx_stream stream);

/* One tensor of a multi-tensor quantization: the arguments of mx_quantize, same meaning. */
typedef struct {
    const void* x;            /* BF16 [M, K], row stride ld_x elements (device) */
    int64_t M, K, ld_x;
    uint8_t* q_row;           /* outputs of the requested directions (device) */
    uint8_t* s_row;
    uint8_t* q_col;
    uint8_t* s_col;
} mx_quant_tensor;

/*
 * mx_quantize over a list of tensors with the same flags, in as few launches as possible (one per
 * 192 tensors). At every weight synchronization the learner quantizes every weight of the model
 * (Figure 1); walking all tensors' tiles as one tile space removes the per-launch ramp and tail.
 * `tensors` is host memory, read during the call. Every tensor is checked as by mx_quantize before
 * anything is launched; the first failing check's status is returned. Results are identical to
 * one mx_quantize call per tensor. Outputs of different tensors must not overlap.
 */
mx_status mx_quantize_multi(const mx_quant_tensor* tensors, int64_t n, int flags, mx_stream stream);

/*
 * Scale rearrangement (Table 6, "scale rearrangement"; Table 10 F3, the interleaved scale copy a
 * backend derives): raw scales s[rows, kblocks] (device, packed) -> the tensor-core layout in
 * s_swz (device). With group_rows_host == NULL the whole matrix is one group
 * (mx_swizzled_scale_bytes(rows, kblocks) bytes). Otherwise group_rows_host (host memory, read
 * during the call) lists `groups` consecutive row counts summing to `rows`; every group is padded
 * to a multiple of 128 rows on its own and the groups' layouts are concatenated
 * (sum_g ceil(rows_g/128)*128 * ceil(kblocks/4)*4 bytes) -- the A-operand scale layout that
 * mx_grouped_gemm reads. Pad bytes are written 0. rows == 0 or kblocks == 0 is a no-op (pointers
 * may then be NULL). Errors: MX_ERR_ARG (negative sizes or group rows, groups < 1 with a list,
 * NULL pointers), MX_ERR_SHAPE (group rows not summing to rows), MX_ERR_ALIGN (s_swz not 16-byte
 * aligned).
 */
mx_status mx_swizzle_scales(const uint8_t* s, int64_t rows, int64_t kblocks,
                            const int64_t* group_rows_host, int64_t groups, uint8_t* s_swz,
                            mx_stream stream);

/*
 * Dense block-scaled MXFP8 GEMM (Table 6, "GEMM"): C[M, N] = A . B^T with
 * A[m, k] = dec(qa[m, k]) * 2^(sa[m, k/32] - 127) and B[n, k] likewise, accumulated in fp32 on
 * the tensor cores and written as fp32 or BF16 (round-to-nearest-even).
 *   qa[M, K], qb[N, K]: E4M3 codes, K-major, packed (device);
 *   sa_swz, sb_swz: scales of qa and qb in the tensor-core layout (as mx_quantize with
 *                   MX_SWIZZLE writes them) (device);
 *   c: device, row stride ld_c elements; rows >= M / columns >= N are never written.
 * Requirements: M, N >= 0, K > 0, K % 32 == 0, ld_c >= N, qa/sa_swz/qb/sb_swz 16-byte aligned,
 * c aligned to its element size, M, N, K < 2^31. Rows of C that start 16-byte aligned (c and
 * ld_c * sizeof(out) multiples of 16) are written with 16-byte stores, others element by element.
 * M == 0 or N == 0 is a no-op (pointers may then be NULL).
 * Accuracy: |c - exact| <= 1e-5 * sum_k |a_k b_k| (+ 2^-8 |exact| for BF16 output).
 */
mx_status mx_gemm(const uint8_t* qa, const uint8_t* sa_swz, const uint8_t* qb, const uint8_t* sb_swz,
                  int64_t M, int64_t N, int64_t K, void* c, int64_t ld_c, mx_out_dtype out_dtype,
                  mx_stream stream);

/*
 * Grouped block-scaled MXFP8 GEMM for MoE experts (Table 2: Qwen3-30B-A3B, 128 experts, top-8;
 * Table 10 F4, the sampler's expert layout). For every group g, rows [off[g], off[g+1]) of A
 * are multiplied with expert weight B_g:  C[r, :] = A[r, :] . B_g^T.
 *   qa[total_rows, K]: E4M3 codes, rows grouped by expert (device);
 *   sa_swz: A's scales in the grouped tensor-core layout (mx_swizzle_scales with the groups'
 *           row counts: each group padded to 128 rows) (device);
 *   qb[G, N, K]: expert weights (device); sb_swz: G consecutive tensor-core layouts of the
 *           experts' [N, K/32] scales, mx_swizzled_scale_bytes(N, K/32) bytes each (device);
 *   row_offsets_dev[G + 1]: int32 device array, 0 = off[0] <= off[1] <= ... <= off[G] =
 *           total_rows. The host never reads it; invalid offsets set a device error bit and no
 *           output is written;
 *   c: device, [total_rows, N] with row stride ld_c.
 * Requirements: 1 <= G <= 1024 and those of mx_gemm.
 */
mx_status mx_grouped_gemm(const uint8_t* qa, const uint8_t* sa_swz, const uint8_t* qb,
                          const uint8_t* sb_swz, const int32_t* row_offsets_dev, int64_t G,
                          int64_t total_rows, int64_t N, int64_t K, void* c, int64_t ld_c,
                          mx_out_dtype out_dtype, mx_stream stream);

/*
 * The expert MLP's first GEMM with its activation and the down GEMM's quantization fused into the
 * epilogue (Table 2: Qwen3-30B-A3B experts, whose down projection consumes this activation in
 * MXFP8). For every group g and row r in [off[g], off[g+1]), with gu = A[r, :] . B_g^T:
 *   h[r, f] = silu(gate[r, f]) * up[r, f],  silu(x) = x / (1 + exp(-x)),  f < n_inter,
 * computed in fp32 from the fp32 accumulator, then quantized rowwise like mx_quantize does a
 * BF16 tensor (32-blocks along f; E8M0 scale from the block's fp32 amax, e = floor(log2 amax) - 8
 * clamped to [-127, 127]; codes RNE(h * 2^-e) saturated to +-448; 0xFF scale and sign|0x7F codes
 * for a block holding NaN or Inf). No BF16 gate_up or h is written.
 *   qa, sa_swz, row_offsets_dev, G, total_rows, K: as mx_grouped_gemm;
 *   qb[G, 2 n_inter, K], sb_swz: the experts' gate and up weights with their rows interleaved per
 *           128: rows [256 t, 256 t + 128) of expert g are gate rows [128 t, 128 t + 128), rows
 *           [256 t + 128, 256 t + 256) the up rows of the same features; scales as mx_grouped_gemm;
 *   h_q[total_rows, n_inter]: E4M3 codes (device, packed);
 *   h_s_swz: h's scales in the grouped tensor-core layout (each group padded to 128 rows; the size
 *           mx_swizzle_scales gives for [total_rows, n_inter / 32] with the groups' row counts),
 *           pad bytes written 0 -- the A-operand scales mx_grouped_gemm reads for the down GEMM.
 * Requirements: n_inter % 128 == 0, h_q and h_s_swz 16-byte aligned, and those of
 * mx_grouped_gemm. Always runs the CTA-pair kernel.
 * Accuracy: h differs from the exact value by the GEMM's error propagated through SwiGLU plus
 * the error of CUDA's __expf and __fdividef (a few ulps, growing with |gate|) and the fp32
 * products, so a code can differ from the exactly
 * rounded one where h lies that close to a rounding boundary, and a scale where the block's amax
 * lies that close to a power of two.
 */
mx_status mx_grouped_gemm_swiglu_quant(const uint8_t* qa, const uint8_t* sa_swz, const uint8_t* qb,
                                       const uint8_t* sb_swz, const int32_t* row_offsets_dev, int64_t G,
                                       int64_t total_rows, int64_t n_inter, int64_t K, uint8_t* h_q,
                                       uint8_t* h_s_swz, mx_stream stream);

/*
 * FP8 blockwise quantization with one scale per 128 x 128 block (Table 1: the FP8-blockwise
 * learner/sampler pairing, whose scales differ on SM100 -- power-of-two for the learner, FP32 for
 * the sampler; Table 10 F6), to measure that pairing's grid gap beside the shared MXFP8 grid.
 * amax = max |x| over the block. pow2_scales == 0: s = fl32(amax / 448) and codes
 * RNE_E4M3(fl32(x / s)) saturated to +-448 (IEEE single divisions). pow2_scales != 0: s = the
 * smallest power of two >= fl32(amax / 448) and codes RNE_E4M3(x / s). An all-zero block takes
 * s = 1; a block holding NaN or Inf takes s = NaN and codes sign|0x7F.
 *   x: BF16 [M, K] (device), row stride ld_x elements; q: [M, K] E4M3 codes (device, packed);
 *   scales: fp32 [ceil(M/128), ceil(K/128)] row-major (device).
 * Requirements: K % 32 == 0, M, K < 2^31 (else MX_ERR_SHAPE), ld_x >= K, ld_x % 8 == 0, x and q
 * 16-byte aligned, scales 4-byte aligned. M == 0 or K == 0 is a no-op (pointers may then be NULL).
 * Errors: MX_ERR_ARG, MX_ERR_SHAPE, MX_ERR_ALIGN as stated; MX_ERR_CUDA on a failed launch.
 */
mx_status mx_quantize_block128(const void* x, int64_t M, int64_t K, int64_t ld_x, int pow2_scales, uint8_t* q,
                               float* scales, mx_stream stream);

/*
 * Selects the kernel behind later mx_gemm / mx_grouped_gemm calls (process-wide): 0 (default) the
 * CTA-pair kernel (256 x 256 tiles computed by two SMs with tcgen05.mma.cta_group::2), 1 the
 * single-CTA kernel (128 x 256 tiles). Both meet the accuracy bound above; results may differ in
 * fp32 summation order only. Other values select 0.
 */
void mx_set_gemm_variant(int variant);

/*
 * Selects the quantizer kernel behind later mx_quantize / mx_quantize_multi calls (process-wide):
 * 0 (default) loads each thread's two 32-element blocks of a 128 x 128 BF16 tile into registers
 * with 256-bit loads, one tile ahead of the compute (the columnwise pass of a row + col call goes
 * through a swizzled shared-memory copy of the tile), except that columnwise-only calls take the
 * TMA-staged kernel, and rowwise-only calls whose CTAs each walk many tiles (at least 64) take a
 * split-load form that loads each half of the next tile as soon as the same half of the current
 * one is encoded; 1 stages the tiles of every call in shared memory with TMA tensor loads running
 * three tiles ahead; 2 is 0 with the split-load form for every rowwise-only call. All produce the
 * same bytes; the default picks the kernel measured faster on B200 for each direction and size.
 * Other values select 0.
 */
void mx_set_quantize_variant(int variant);

/*
 * Byte comparison (abstract and Table 11: the synchronized sampler weights, scales and kernel
 * layout must equal the learner's quantization byte for byte): counts the positions i < nbytes
 * with a[i] != b[i] and finds the smallest such i. Results are written to device memory:
 * *mismatches_dev (uint64) and *first_index_dev (int64, -1 if none); both are overwritten.
 * a, b: device buffers (any alignment; 16-byte aligned ones take the vector path).
 */
mx_status mx_grid_equal(const uint8_t* a, const uint8_t* b, int64_t nbytes,
                        unsigned long long* mismatches_dev, long long* first_index_dev,
                        mx_stream stream);

/* One pair of a multi-pair byte comparison. */
typedef struct {
    const uint8_t* a;         /* device */
    const uint8_t* b;         /* device */
    int64_t nbytes;
} mx_compare_pair;

/*
 * mx_grid_equal over n pairs in one pass (the byte comparison of a whole synchronization: every
 * weight's elements, raw scales and swizzled scales). For pair i, mismatches_dev[i] (uint64) and
 * first_index_dev[i] (int64, -1 if equal) are written (device arrays of n entries each). `pairs`
 * is host memory, read during the call. Results are identical to n mx_grid_equal calls.
 */
mx_status mx_grid_equal_multi(const mx_compare_pair* pairs, int64_t n, unsigned long long* mismatches_dev,
                              long long* first_index_dev, mx_stream stream);

/* The grid a quantization is compared with in mx_quantize_compare_multi. */
typedef struct {
    const uint8_t* q;         /* codes [M, K] (device, 16-byte aligned) */
    const uint8_t* s;         /* scales in the tensor-core layout (device, 16-byte aligned) */
} mx_grid_ref;

/*
 * Weight synchronization in one pass (Figure 1: the learner quantizes its weights; Table 11: the
 * sampler's copy must equal them byte for byte): mx_quantize_multi(tensors, n, MX_ROWWISE |
 * MX_SWIZZLE) -- the same codes and layout bytes are written to each tensor's q_row / s_row --
 * fused with the byte comparison of what it writes against refs[i] (e.g. the sampler's copy),
 * which is read once instead of comparing the written grid in a second pass. Results, on the
 * device, as mx_grid_equal_multi gives them for the pairs (q_row_i, refs[i].q) and
 * (s_row_i, refs[i].s): mismatches_dev[2i] / first_index_dev[2i] for the codes (M*K bytes) and
 * [2i + 1] for the scale layout (mx_swizzled_scale_bytes(M, K/32) bytes); -1 if equal. Entries of
 * tensors with M == 0 or K == 0 report 0 / -1. `tensors` and `refs` are host memory, read during
 * the call; each tensor is checked as by mx_quantize (q_col / s_col ignored). Errors: MX_ERR_ARG
 * (NULL arrays or reference pointers, n < 0 or n > 2^30), MX_ERR_ALIGN (reference not 16-byte
 * aligned), and those of mx_quantize.
 */
mx_status mx_quantize_compare_multi(const mx_quant_tensor* tensors, const mx_grid_ref* refs, int64_t n,
                                    unsigned long long* mismatches_dev, long long* first_index_dev,
                                    mx_stream stream);

/* Human-readable name of a status code (static string). */
const char* mx_status_string(mx_status status);

/*
 * Reads and clears the device status word of the current device (synchronizes the device).
 * *bits receives the error bits (1: a bounded wait expired; 2: invalid grouped-GEMM row offsets).
 * Returns MX_OK when no bit was set, MX_ERR_DEVICE when some bit was set, MX_ERR_CUDA on failure.
 */
mx_status mx_device_error(uint32_t* bits);

/*
 * Deadline of every bounded wait inside libmx kernels, in nanoseconds (default 2e9 = 2 s); 0
 * restores the default. Affects launches made after the call. After a wait expires, a kernel still
 * waits for its own copies and MMAs in flight before it exits; those drain waits take at least 1 s
 * whatever this deadline is.
 */
void mx_set_wait_timeout_ns(uint64_t ns);

/*
 * Diagnostic: launches one block whose thread waits on an mbarrier that nothing ever completes,
 * under the current wait deadline. The wait expires, the kernel records error bit 1 and
 * returns; read it with mx_device_error. Used to test that expired waits end a kernel cleanly.
 */
mx_status mx_diag_expired_wait(mx_stream stream);

#ifdef __cplusplus
}
#endif
#endif /* MX_H */
