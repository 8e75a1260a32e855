/*
 * CPU oracle for the MXFP8 learner/sampler grid -- TEST INFRASTRUCTURE ONLY.
 * (Only tests/, __graft_entry__.smoke() and bench.py's CPU baseline use it; the CUDA
 * library never does.) See mx_oracle.h for the sources each function follows.
 *
 * Plain fp64 loops, single-threaded, no code shared with the GPU path.
 */
#include "mx_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ---- element formats ---------------------------------------------------------------- */

/* BF16 is the upper half of an IEEE binary32; widening to double is exact. */
static double bf16_to_double(uint16_t bits) {
    uint32_t w = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

/* E4M3 "fn" encoding (OCP 8-bit floating point, E4M3 variant): sign bit, 4 exponent bits
 * with bias 7, 3 mantissa bits, no infinities, S.1111.111 = NaN, largest finite 448,
 * subnormals (exponent field 0) of value mantissa * 2^-9. */
double oracle_e4m3_decode(uint8_t code) {
    int sign = code >> 7;
    int expo = (code >> 3) & 0xF;
    int mant = code & 0x7;
    double v;
    if (expo == 0xF && mant == 0x7) return NAN;
    if (expo == 0)
        v = ldexp((double)mant, -9);
    else
        v = ldexp(1.0 + mant / 8.0, expo - 7);
    return sign ? -v : v;
}

/* Round to nearest, ties to even, onto the E4M3 grid; magnitudes above 448 saturate to 448
 * (no NaN is produced from a finite input). The sign of zero is kept. */
uint8_t oracle_e4m3_encode(double v) {
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs(v);
    if (a == 0.0) return sign;

    /* Spacing of the grid around a: 2^(E-3) in the binade [2^E, 2^(E+1)) for E >= -6;
     * the subnormal range below 2^-6 has the spacing of the lowest normal binade, 2^-9. */
    int ex;
    frexp(a, &ex);           /* a = f * 2^ex, f in [0.5, 1) -> floor(log2 a) = ex - 1 */
    int E = ex - 1;
    if (E < -6) E = -6;
    double quantum = ldexp(1.0, E - 3);
    double r = a / quantum;  /* exact: division by a power of two */
    double fl = floor(r);
    double frac = r - fl;
    double n = fl;
    if (frac > 0.5 || (frac == 0.5 && fmod(fl, 2.0) == 1.0)) n = fl + 1.0;
    double value = n * quantum;
    if (value > 448.0) value = 448.0;   /* saturate to the largest finite E4M3 value */
    if (value == 0.0) return sign;

    /* Encode the (now representable) value. */
    frexp(value, &ex);
    E = ex - 1;
    uint8_t mag;
    if (E < -6) {
        mag = (uint8_t)(value / ldexp(1.0, -9));            /* subnormal: mantissa only */
    } else {
        int mant = (int)((value / ldexp(1.0, E) - 1.0) * 8.0);
        mag = (uint8_t)(((E + 7) << 3) | mant);
    }
    return sign | mag;
}

void oracle_e4m3_encode_array(const double* v, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(v[i]);
}

/* E8M0 shared scale (OCP MX): X = 2^(floor(log2 amax) - 8), 8 being the exponent of the
 * largest power of two in E4M3 (448 = 1.75 * 2^8). The exponent is clamped to the E8M0
 * range [-127, 127] and stored with bias 127. An all-zero block takes the smallest scale. */
uint8_t oracle_e8m0_scale(double amax) {
    int e;
    if (amax == 0.0) {
        e = -127;
    } else {
        int ex;
        frexp(amax, &ex);
        e = (ex - 1) - 8;
        if (e < -127) e = -127;
        if (e > 127) e = 127;
    }
    return (uint8_t)(e + 127);
}

/* One 32-element block: x[i * stride], i < 32. Writes q[i] and returns the scale byte.
 * NaN/Inf policy (the pages do not fix one): a block holding any NaN or infinity gets the
 * E8M0 NaN scale 0xFF and every element byte is sign | 0x7F (the E4M3 NaN). */
static uint8_t quantize_block(const uint16_t* x, int64_t stride, uint8_t* q, int64_t qstride) {
    double v[32];
    int special = 0;
    double amax = 0.0;
    for (int i = 0; i < 32; ++i) {
        v[i] = bf16_to_double(x[i * stride]);
        if (isnan(v[i]) || isinf(v[i])) special = 1;
        else if (fabs(v[i]) > amax) amax = fabs(v[i]);
    }
    if (special) {
        for (int i = 0; i < 32; ++i) q[i * qstride] = (uint8_t)((signbit(v[i]) ? 0x80 : 0) | 0x7F);
        return 0xFF;
    }
    uint8_t s = oracle_e8m0_scale(amax);
    int e = (int)s - 127;
    for (int i = 0; i < 32; ++i) q[i * qstride] = oracle_e4m3_encode(ldexp(v[i], -e));  /* exact */
    return s;
}

int oracle_quantize_rowwise(const uint16_t* x, int64_t M, int64_t K, int64_t ld,
                            uint8_t* q, uint8_t* s) {
    if (K % 32 != 0) return -1;
    int64_t nb = K / 32;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t b = 0; b < nb; ++b)
            s[m * nb + b] = quantize_block(x + m * ld + b * 32, 1, q + m * K + b * 32, 1);
    return 0;
}

int oracle_quantize_colwise(const uint16_t* x, int64_t M, int64_t K, int64_t ld,
                            uint8_t* qT, uint8_t* sT) {
    if (M % 32 != 0) return -1;
    /* The columnwise copy is the rowwise quantization of the transpose: build x^T [K, M]. */
    uint16_t* xt = (uint16_t*)malloc((size_t)(M * K > 0 ? M * K : 1) * sizeof(uint16_t));
    if (!xt) return -2;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k) xt[k * M + m] = x[m * ld + k];
    int rc = oracle_quantize_rowwise(xt, K, M, M, qT, sT);
    free(xt);
    return rc;
}

void oracle_dequantize(const uint8_t* q, const uint8_t* s, int64_t rows, int64_t K, double* out) {
    int64_t nb = K / 32;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t sb = s[r * nb + k / 32];
            double scale = (sb == 0xFF) ? NAN : ldexp(1.0, (int)sb - 127);
            out[r * K + k] = oracle_e4m3_decode(q[r * K + k]) * scale;
        }
}

/* ---- scale layout --------------------------------------------------------------------- */

static int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

int64_t oracle_swizzled_size(int64_t rows, int64_t cols, const int64_t* group_rows,
                             int64_t groups) {
    int64_t padded_cols = round_up(cols, 4);
    if (!group_rows) return round_up(rows, 128) * padded_cols;
    int64_t total = 0;
    for (int64_t g = 0; g < groups; ++g) total += round_up(group_rows[g], 128) * padded_cols;
    return total;
}

/* Tensor-core scale-factor layout (NVIDIA sm_100 block-scaling-factor layout): the padded
 * [R', C'] scale matrix is cut into 128-row x 4-column blocks stored one after another
 * (row-block major, then column-block), 512 bytes each; inside a block, scale (r, c) sits at
 * byte (r % 32) * 16 + (r / 32) * 4 + c. */
void oracle_swizzle(const uint8_t* s, int64_t rows, int64_t cols, const int64_t* group_rows,
                    int64_t groups, uint8_t* out) {
    int64_t padded_cols = round_up(cols, 4);
    int64_t one_group = rows;
    if (!group_rows) { group_rows = &one_group; groups = 1; }
    memset(out, 0, (size_t)oracle_swizzled_size(rows, cols, group_rows, groups));
    int64_t src_row = 0, dst_base = 0;
    for (int64_t g = 0; g < groups; ++g) {
        int64_t n = group_rows[g];
        for (int64_t r = 0; r < n; ++r)
            for (int64_t c = 0; c < cols; ++c) {
                int64_t block = (r / 128) * (padded_cols / 4) + c / 4;
                int64_t inner = (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4);
                out[dst_base + block * 512 + inner] = s[(src_row + r) * cols + c];
            }
        src_row += n;
        dst_base += round_up(n, 128) * padded_cols;
    }
}

/* ---- block-scaled GEMM ------------------------------------------------------------------ */

static double dq(uint8_t code, uint8_t scale) {
    if (scale == 0xFF) return NAN;
    return oracle_e4m3_decode(code) * ldexp(1.0, (int)scale - 127);
}

/* Every product of two dequantized MXFP8 values is exact in fp64 (at most 8 significant
 * bits, exponent >= -290); the sum is taken in fp64 in k order. */
void oracle_gemm(const uint8_t* qa, const uint8_t* sa, const uint8_t* qb, const uint8_t* sb,
                 int64_t M, int64_t N, int64_t K, double* c, double* abs_sum) {
    int64_t nb = K / 32;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0, acc_abs = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double p = dq(qa[m * K + k], sa[m * nb + k / 32]) * dq(qb[n * K + k], sb[n * nb + k / 32]);
                acc += p;
                acc_abs += fabs(p);
            }
            c[m * N + n] = acc;
            if (abs_sum) abs_sum[m * N + n] = acc_abs;
        }
}

void oracle_grouped_gemm(const uint8_t* qa, const uint8_t* sa, const uint8_t* qb,
                         const uint8_t* sb, const int64_t* row_offsets, int64_t groups,
                         int64_t N, int64_t K, double* c, double* abs_sum) {
    int64_t nb = K / 32;
    for (int64_t g = 0; g < groups; ++g) {
        int64_t r0 = row_offsets[g], r1 = row_offsets[g + 1];
        oracle_gemm(qa + r0 * K, sa + r0 * nb, qb + g * N * K, sb + g * N * nb,
                    r1 - r0, N, K, c + r0 * N, abs_sum ? abs_sum + r0 * N : NULL);
    }
}

/* ---- FP8 blockwise, 128 x 128 blocks, FP32 or power-of-two scales -------------------------- */

void oracle_quantize_block128(const uint16_t* x, int64_t M, int64_t K, int64_t ld, int pow2, uint8_t* q,
                              float* scales) {
    const int64_t bm = (M + 127) / 128, bk = (K + 127) / 128;
    for (int64_t i = 0; i < bm; ++i) {
        for (int64_t j = 0; j < bk; ++j) {
            const int64_t r1 = (i + 1) * 128 < M ? (i + 1) * 128 : M;
            const int64_t c1 = (j + 1) * 128 < K ? (j + 1) * 128 : K;
            double amax = 0.0;
            int special = 0;
            for (int64_t r = i * 128; r < r1; ++r)
                for (int64_t c = j * 128; c < c1; ++c) {
                    const double v = bf16_to_double(x[r * ld + c]);
                    if (isnan(v) || isinf(v)) special = 1;
                    else if (fabs(v) > amax) amax = fabs(v);
                }
            float s;
            if (special) {
                s = NAN;
            } else if (amax == 0.0) {
                s = 1.0f;
            } else {
                s = (float)amax / 448.0f;                  /* IEEE single division */
                if (pow2) {
                    const int e = ilogbf(s);
                    const float p = ldexpf(1.0f, e);
                    s = (p == s) ? p : ldexpf(1.0f, e + 1);
                }
            }
            scales[i * bk + j] = s;
            for (int64_t r = i * 128; r < r1; ++r)
                for (int64_t c = j * 128; c < c1; ++c) {
                    const float v = (float)bf16_to_double(x[r * ld + c]);
                    if (special) {
                        q[r * K + c] = (uint8_t)((signbit(v) ? 0x80 : 0) | 0x7F);
                    } else {
                        const float t = v / s;                /* IEEE single division */
                        q[r * K + c] = oracle_e4m3_encode((double)t);
                    }
                }
        }
    }
}

/* ---- SwiGLU activation + MXFP8 rule (fp64) -------------------------------------------------- */

static double silu(double x) { return x / (1.0 + exp(-x)); }

int oracle_swiglu_quantize(const double* gu, int64_t rows, int64_t n, double* h, uint8_t* q, uint8_t* s) {
    if (n % 32 != 0) return -1;
    double v[32];
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < n / 32; ++b) {
            double amax = 0.0;
            int special = 0;
            for (int i = 0; i < 32; ++i) {
                const int64_t f = b * 32 + i;
                v[i] = silu(gu[r * 2 * n + f]) * gu[r * 2 * n + n + f];
                if (h) h[r * n + f] = v[i];
                if (isnan(v[i]) || isinf(v[i])) special = 1;
                else if (fabs(v[i]) > amax) amax = fabs(v[i]);
            }
            uint8_t* qb = q + r * n + b * 32;
            if (special) {
                /* same NaN/Inf policy as the BF16 quantizer */
                for (int i = 0; i < 32; ++i) qb[i] = (uint8_t)((signbit(v[i]) ? 0x80 : 0) | 0x7F);
                s[r * (n / 32) + b] = 0xFF;
                continue;
            }
            const uint8_t sc = oracle_e8m0_scale(amax);
            const int e = (int)sc - 127;
            for (int i = 0; i < 32; ++i) qb[i] = oracle_e4m3_encode(ldexp(v[i], -e));
            s[r * (n / 32) + b] = sc;
        }
    }
    return 0;
}

/* ---- byte comparison ---------------------------------------------------------------------- */

void oracle_grid_equal(const uint8_t* a, const uint8_t* b, int64_t nbytes,
                       uint64_t* mismatches, int64_t* first_index) {
    uint64_t count = 0;
    int64_t first = -1;
    for (int64_t i = 0; i < nbytes; ++i)
        if (a[i] != b[i]) {
            if (first < 0) first = i;
            ++count;
        }
    *mismatches = count;
    *first_index = first;
}
