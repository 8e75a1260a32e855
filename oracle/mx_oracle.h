/*
 * CPU oracle for the MXFP8 learner/sampler grid -- TEST INFRASTRUCTURE ONLY.
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline leg (and its
 * `--impl reference` arm) may load this library. The product library (libmx) never
 * links, includes or calls it, and it shares no code with the CUDA path.
 *
 * Source: "End-to-End MXFP8 Reinforcement Learning on Blackwell: What Matching Buys,
 * When It Pays Off, and How It Fails" (W. Zhang, arXiv 2610.34915), as printed on
 * thelatestinai.com/papers/2610.34915:
 *   - Figure 1: the learner quantizes BF16 master weights with its own quantizer and the
 *     sampler receives that grid, then re-derives its kernel layouts;
 *   - Table 1: on SM100 the block scales are powers of two;
 *   - Table 10 (F6): E8M0 scales keep only the exponent;
 *   - Table 10 (F3): the backend derives an interleaved scale copy (the swizzle);
 *   - Table 11 (byte comparison): sampler weight, scale and kernel layout must equal the
 *     learner's quantization byte for byte.
 * The pages do not print the quantization rule itself; it is the OCP Microscaling (MX)
 * v1.0 rule for MXFP8 (E4M3 elements, E8M0 shared scale, 32-element blocks):
 * scale exponent = floor(log2(amax)) - emax_elem (8 for E4M3), clamped to the E8M0 range.
 * The scale-factor layout is NVIDIA's published sm_100 block-scaling-factor layout
 * (128x4 blocks of scales, 512 bytes each); it is not on the pages either.
 *
 * Arithmetic is fp64 throughout. Every function is a plain loop; no blocking, no
 * fusion, no reordering beyond what the definition states.
 */
#ifndef MX_ORACLE_H
#define MX_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exact value of one FP8 E4M3 (fn variant) code; NaN for S.1111.111. */
double oracle_e4m3_decode(uint8_t code);
/* Round-to-nearest-even onto the E4M3 grid, saturating |v| > 448 to 448. v must be finite. */
uint8_t oracle_e4m3_encode(double v);
/* oracle_e4m3_encode over an array (for exhaustive tests). */
void oracle_e4m3_encode_array(const double* v, int64_t n, uint8_t* out);
/* E8M0 scale byte for one block whose largest magnitude is amax (finite, >= 0). */
uint8_t oracle_e8m0_scale(double amax);

/* Rowwise MXFP8 quantization of a BF16 matrix x[M, K] (row stride ld elements),
 * one scale per 32 consecutive elements along K.
 * q[M, K] (packed, row stride K), s[M, K/32] (packed). Returns 0, or -1 if K % 32 != 0. */
int oracle_quantize_rowwise(const uint16_t* x, int64_t M, int64_t K, int64_t ld,
                            uint8_t* q, uint8_t* s);
/* Columnwise quantization: by definition the rowwise quantization of x^T.
 * qT[K, M], sT[K, M/32]. Returns 0, or -1 if M % 32 != 0. */
int oracle_quantize_colwise(const uint16_t* x, int64_t M, int64_t K, int64_t ld,
                            uint8_t* qT, uint8_t* sT);
/* Dequantize: out[r, k] = decode(q[r, k]) * 2^(s[r, k/32] - 127), fp64. */
void oracle_dequantize(const uint8_t* q, const uint8_t* s, int64_t rows, int64_t K,
                       double* out);

/* Size in bytes of the tensor-core scale layout for a [rows, cols] scale matrix split into
 * groups of group_rows[g] rows (group_rows == NULL means one group of `rows`). */
int64_t oracle_swizzled_size(int64_t rows, int64_t cols, const int64_t* group_rows,
                             int64_t groups);
/* Scale rearrangement into 128x4 blocks of 512 bytes; each group padded to 128 rows and
 * the columns padded to a multiple of 4; pad bytes are 0. */
void oracle_swizzle(const uint8_t* s, int64_t rows, int64_t cols, const int64_t* group_rows,
                    int64_t groups, uint8_t* out);

/* Block-scaled GEMM with raw (unswizzled) scales:
 * c[m, n] = sum_k dq(qa[m,k]) * dq(qb[n,k]); abs_sum[m, n] = sum_k |dq(qa) * dq(qb)|.
 * qa[M, K], sa[M, K/32], qb[N, K], sb[N, K/32]; abs_sum may be NULL. */
void oracle_gemm(const uint8_t* qa, const uint8_t* sa, const uint8_t* qb, const uint8_t* sb,
                 int64_t M, int64_t N, int64_t K, double* c, double* abs_sum);
/* Grouped GEMM: rows [off[g], off[g+1]) of A against expert weight B_g = qb[g] ([N, K]).
 * c[total_rows, N]. */
void oracle_grouped_gemm(const uint8_t* qa, const uint8_t* sa, const uint8_t* qb,
                         const uint8_t* sb, const int64_t* row_offsets, int64_t groups,
                         int64_t N, int64_t K, double* c, double* abs_sum);

/* FP8 blockwise quantization with one scale per 128 x 128 block of a BF16 weight x[M, K] (the
 * "FP8 blockwise" recipe of Table 1, whose learner and sampler differ in their scales on SM100:
 * power-of-two against FP32; Table 10 F6). amax = max |x| over the block. FP32 scales
 * (pow2 == 0): s = fl32(amax / 448); codes RNE_E4M3(fl32(x / s)) saturated to +-448, both
 * divisions in IEEE single precision. Power-of-two scales (pow2 != 0): s = the smallest power of
 * two >= fl32(amax / 448); codes RNE_E4M3(x / s). An all-zero block takes s = 1; a block holding
 * NaN or Inf takes s = NaN and codes sign | 0x7F. q[M, K]; scales[ceil(M/128), ceil(K/128)] fp32.
 * Edge blocks cover what exists. */
void oracle_quantize_block128(const uint16_t* x, int64_t M, int64_t K, int64_t ld, int pow2, uint8_t* q,
                              float* scales);

/* The MoE expert MLP's activation between its two GEMMs, then the MXFP8 rule on the result
 * (Table 2: Qwen3-30B-A3B experts; the down projection consumes this activation quantized):
 *   h[r, f] = silu(gu[r, f]) * gu[r, n + f],  silu(x) = x / (1 + exp(-x)),  f < n,
 * from the gate_up product gu [rows, 2n] (gate features first, then up features), all in fp64.
 * Each row of h is then quantized in 32-blocks exactly as a rowwise BF16 tensor would be
 * (same scale rule, same rounding), from the fp64 values. Writes h (fp64, may be NULL),
 * q [rows, n] and raw scales s [rows, n / 32]. Returns -1 if n % 32 != 0. */
int oracle_swiglu_quantize(const double* gu, int64_t rows, int64_t n, double* h, uint8_t* q, uint8_t* s);

/* Byte comparison: number of positions i with a[i] != b[i] and the first such i (-1 if none). */
void oracle_grid_equal(const uint8_t* a, const uint8_t* b, int64_t nbytes,
                       uint64_t* mismatches, int64_t* first_index);

#ifdef __cplusplus
}
#endif
#endif
