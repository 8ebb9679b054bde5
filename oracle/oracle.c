/*
 * oracle.c -- plain, slow CPU oracle for block-quantized dequantize + GEMV.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke entry and
 * the benchmark's CPU-baseline leg may load this library.  The CUDA library
 * never links, calls or falls back to it, and this file shares no code, header,
 * table or constant with it.
 *
 * Everything here is the plain definition of the operation, written out in
 * double precision, one weight at a time, with no blocking, fusion or
 * reordering:
 *
 *   - GGML-style block formats, as used by the pages' "upload raw Q4K weight
 *     bytes for fused dequant+GEMV" entry point (trueno WgslForwardPass,
 *     upload_q4k_weight) and by the CUDA lane's Q8_0 GEMV and its CPU oracle
 *     (qualiaDB cuda_lane module map: try_q8_0_cuda_gemv,
 *     q8_0_gemv_oracle_into, Q8_0_BLOCK_BYTES, Q8_0_BLOCK_ELEMS).
 *       Q8_0 block, 34 bytes, 32 weights:  [d: fp16][q: 32 x int8]
 *       Q4_K super-block, 144 bytes, 256 weights:
 *                 [d: fp16][dmin: fp16][scales: 12 bytes][qs: 128 bytes]
 *     Bytes are little-endian.  A row of K weights is K/32 (Q8_0) or K/256
 *     (Q4_K) consecutive blocks; rows follow each other with no padding.
 *   - GEMV y[b][n] = sum_k W[n][k] * x[b][k], accumulated in double over the
 *     exact (double) dequantized weights, together with the error scale
 *     A[b][n] = sum_k |W[n][k] * x[b][k]| that the tolerance rule uses.
 *   - The fused gate/up variant silu(W_g x) * (W_u x) (qualiaDB cuda_lane:
 *     try_q4k_soa_fused_swiglu; trueno WgslForwardPass: silu_mul_shader).
 *   - The structure-of-arrays repack (qualiaDB cuda_lane:
 *     preload_q4k_soa_weights / try_q4k_soa_gemv).  The pages name the SoA
 *     layout but do not define it; the layout below is this library's own and
 *     is written out in full next to oracle_q4k_repack_soa.
 *
 * No function here may fail on well-formed input.  Functions that take sizes
 * return 0 on success and a negative number when the sizes are malformed.
 */

#include <math.h>
#include <stdint.h>
#include <stddef.h>

#define Q8_0_BLOCK_ELEMS 32
#define Q8_0_BLOCK_BYTES 34
#define Q4K_BLOCK_ELEMS 256
#define Q4K_BLOCK_BYTES 144
#define Q4K_SOA_GROUP 4

/* ------------------------------------------------------------------------ */
/* IEEE 754 binary16 -> double.  1 sign bit, 5 exponent bits (bias 15),     */
/* 10 mantissa bits.  Exponent 0 is the subnormal range m * 2^-24; exponent */
/* 31 is Inf (m == 0) or NaN.  Every binary16 value is exact in double.     */
/* ------------------------------------------------------------------------ */
double oracle_fp16_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 31;
    int m = h & 1023;
    double v;
    if (e == 0) {
        v = ldexp((double)m, -24);
    } else if (e == 31) {
        v = (m == 0) ? INFINITY : NAN;
    } else {
        /* (1 + m/1024) * 2^(e-15) */
        v = ldexp(1024.0 + (double)m, e - 15 - 10);
    }
    return sign ? -v : v;
}

static double read_fp16(const uint8_t *p)
{
    uint16_t h = (uint16_t)p[0] | (uint16_t)((uint16_t)p[1] << 8);
    return oracle_fp16_to_double(h);
}

/* Bits [lo, lo+n) of one byte, as an unsigned integer. */
static int bits_of(uint8_t byte, int lo, int n)
{
    return (byte >> lo) & ((1 << n) - 1);
}

/* ------------------------------------------------------------------------ */
/* Q4_K 6-bit scale/min fields (GGML get_scale_min_k4 packing).  The 12     */
/* bytes s[0..11] hold 8 (scale, min) pairs, 16 six-bit fields, 96 bits:    */
/*   j = 0..3: scale_j = bits 0..5 of s[j]                                 */
/*             min_j   = bits 0..5 of s[j+4]                               */
/*   j = 4..7: scale_j = bits 0..3 of s[j+4]  (low 4 bits of the field)    */
/*                     + bits 6..7 of s[j-4]  (high 2 bits of the field)   */
/*             min_j   = bits 4..7 of s[j+4]  (low 4 bits)                 */
/*                     + bits 6..7 of s[j]    (high 2 bits)                */
/* ------------------------------------------------------------------------ */
void oracle_q4k_scale_min(const uint8_t *s, int j, int *scale, int *min)
{
    if (j < 4) {
        *scale = bits_of(s[j], 0, 6);
        *min = bits_of(s[j + 4], 0, 6);
    } else {
        *scale = bits_of(s[j + 4], 0, 4) + 16 * bits_of(s[j - 4], 6, 2);
        *min = bits_of(s[j + 4], 4, 4) + 16 * bits_of(s[j], 6, 2);
    }
}

/* Quant i (0..255) of a Q4_K super-block.  The 128 quant bytes are four    */
/* 32-byte chunks; chunk c covers weights 64c .. 64c+63: the low nibbles of  */
/* its 32 bytes are weights 64c .. 64c+31 (sub-block 2c), the high nibbles   */
/* weights 64c+32 .. 64c+63 (sub-block 2c+1).                                */
int oracle_q4k_quant(const uint8_t *qs, int i)
{
    int c = i / 64;
    int r = i % 64;
    uint8_t byte = qs[32 * c + (r % 32)];
    return (r < 32) ? bits_of(byte, 0, 4) : bits_of(byte, 4, 4);
}

/* One Q4_K super-block (144 bytes) -> 256 exact weights in double:
 *   w_i = d * scale_j * q_i - dmin * min_j,  j = i / 32.
 * d*scale*q has at most 11+6+4 significant bits and dmin*min at most 17, so
 * both products and their difference are exact in double. */
void oracle_q4k_block(const uint8_t *blk, double *w)
{
    double d = read_fp16(blk + 0);
    double dmin = read_fp16(blk + 2);
    const uint8_t *s = blk + 4;
    const uint8_t *qs = blk + 16;
    for (int i = 0; i < Q4K_BLOCK_ELEMS; ++i) {
        int sc, mn;
        oracle_q4k_scale_min(s, i / 32, &sc, &mn);
        int q = oracle_q4k_quant(qs, i);
        w[i] = d * (double)sc * (double)q - dmin * (double)mn;
    }
}

/* One Q8_0 block (34 bytes) -> 32 exact weights: w_i = d * q_i, q_i int8. */
void oracle_q8_0_block(const uint8_t *blk, double *w)
{
    double d = read_fp16(blk);
    for (int i = 0; i < Q8_0_BLOCK_ELEMS; ++i) {
        int q = (int)(int8_t)blk[2 + i];
        w[i] = d * (double)q;
    }
}

/* ------------------------------------------------------------------------ */
/* Structure-of-arrays layout of Q4_K (this library's definition).          */
/*                                                                          */
/* Each row keeps its byte range and its size (144 bytes per super-block).  */
/* Within the row, the super-blocks are taken in groups of 4 consecutive    */
/* blocks (the last group of a row holds the remaining g <= 4 blocks).      */
/* A group of g blocks, starting at byte 144 * 4 * group of the row, is     */
/* stored as                                                                */
/*   g headers of 16 bytes:  header t = bytes 0..15 of block t             */
/*                           (d, dmin, 12 scale bytes)                     */
/*   then for slice s = 0..7: g pieces of 16 bytes:                        */
/*                           piece t = quant bytes qs[16s .. 16s+15] of    */
/*                           block t                                       */
/* so that a group is 16*g + 8*16*g = 144*g bytes.                          */
/* ------------------------------------------------------------------------ */

/* Byte offset, within its row, of AoS byte `byte_in_block` (0..143) of
 * super-block kb, in the SoA layout of a row with nb super-blocks. */
static int64_t soa_offset(int64_t nb, int64_t kb, int byte_in_block)
{
    int64_t group = kb / Q4K_SOA_GROUP;
    int64_t t = kb % Q4K_SOA_GROUP;
    int64_t first = group * Q4K_SOA_GROUP;
    int64_t g = nb - first;
    if (g > Q4K_SOA_GROUP)
        g = Q4K_SOA_GROUP;
    int64_t base = first * Q4K_BLOCK_BYTES;
    if (byte_in_block < 16)
        return base + 16 * t + byte_in_block;
    int qb = byte_in_block - 16;  /* 0..127 */
    int s = qb / 16;
    int within = qb % 16;
    return base + 16 * g + (int64_t)s * 16 * g + 16 * t + within;
}

int oracle_q4k_repack_soa(const uint8_t *aos, int64_t N, int64_t K, uint8_t *soa)
{
    if (N < 0 || K < 0 || K % Q4K_BLOCK_ELEMS != 0)
        return -1;
    int64_t nb = K / Q4K_BLOCK_ELEMS;
    int64_t row_bytes = nb * Q4K_BLOCK_BYTES;
    for (int64_t n = 0; n < N; ++n) {
        const uint8_t *src = aos + n * row_bytes;
        uint8_t *dst = soa + n * row_bytes;
        for (int64_t kb = 0; kb < nb; ++kb)
            for (int b = 0; b < Q4K_BLOCK_BYTES; ++b)
                dst[soa_offset(nb, kb, b)] = src[kb * Q4K_BLOCK_BYTES + b];
    }
    return 0;
}

/* Gathers super-block kb of a row back into AoS order from either layout. */
static void gather_q4k_block(const uint8_t *row, int64_t nb, int64_t kb, int soa,
                             uint8_t *blk)
{
    for (int b = 0; b < Q4K_BLOCK_BYTES; ++b)
        blk[b] = soa ? row[soa_offset(nb, kb, b)] : row[kb * Q4K_BLOCK_BYTES + b];
}

/* ------------------------------------------------------------------------ */
/* Dequantization of whole matrices (N rows x K weights), row-major out.    */
/* ------------------------------------------------------------------------ */
int oracle_q8_0_dequant(const uint8_t *w, int64_t N, int64_t K, double *out)
{
    if (N < 0 || K < 0 || K % Q8_0_BLOCK_ELEMS != 0)
        return -1;
    int64_t nb = K / Q8_0_BLOCK_ELEMS;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t kb = 0; kb < nb; ++kb)
            oracle_q8_0_block(w + (n * nb + kb) * Q8_0_BLOCK_BYTES,
                              out + n * K + kb * Q8_0_BLOCK_ELEMS);
    return 0;
}

int oracle_q4k_dequant(const uint8_t *w, int soa, int64_t N, int64_t K, double *out)
{
    if (N < 0 || K < 0 || K % Q4K_BLOCK_ELEMS != 0)
        return -1;
    int64_t nb = K / Q4K_BLOCK_ELEMS;
    uint8_t blk[Q4K_BLOCK_BYTES];
    for (int64_t n = 0; n < N; ++n) {
        const uint8_t *row = w + n * nb * Q4K_BLOCK_BYTES;
        for (int64_t kb = 0; kb < nb; ++kb) {
            gather_q4k_block(row, nb, kb, soa, blk);
            oracle_q4k_block(blk, out + n * K + kb * Q4K_BLOCK_ELEMS);
        }
    }
    return 0;
}

/* The same values rounded once to the nearest fp32 (ties to even).  The exact
 * weight is a double, so the cast below is the single rounding. */
int oracle_q4k_dequant_f32(const uint8_t *w, int soa, int64_t N, int64_t K, float *out)
{
    if (N < 0 || K < 0 || K % Q4K_BLOCK_ELEMS != 0)
        return -1;
    int64_t nb = K / Q4K_BLOCK_ELEMS;
    uint8_t blk[Q4K_BLOCK_BYTES];
    double tmp[Q4K_BLOCK_ELEMS];
    for (int64_t n = 0; n < N; ++n) {
        const uint8_t *row = w + n * nb * Q4K_BLOCK_BYTES;
        for (int64_t kb = 0; kb < nb; ++kb) {
            gather_q4k_block(row, nb, kb, soa, blk);
            oracle_q4k_block(blk, tmp);
            for (int i = 0; i < Q4K_BLOCK_ELEMS; ++i)
                out[n * K + kb * Q4K_BLOCK_ELEMS + i] = (float)tmp[i];
        }
    }
    return 0;
}

int oracle_q8_0_dequant_f32(const uint8_t *w, int64_t N, int64_t K, float *out)
{
    if (N < 0 || K < 0 || K % Q8_0_BLOCK_ELEMS != 0)
        return -1;
    int64_t nb = K / Q8_0_BLOCK_ELEMS;
    double tmp[Q8_0_BLOCK_ELEMS];
    for (int64_t n = 0; n < N; ++n)
        for (int64_t kb = 0; kb < nb; ++kb) {
            oracle_q8_0_block(w + (n * nb + kb) * Q8_0_BLOCK_BYTES, tmp);
            for (int i = 0; i < Q8_0_BLOCK_ELEMS; ++i)
                out[n * K + kb * Q8_0_BLOCK_ELEMS + i] = (float)tmp[i];
        }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* GEMV on a list of rows.  x is B x K fp32 (row-major); rows[] lists the   */
/* output rows to compute; y and a are B x nrows (row-major):               */
/*   y[b][r] = sum_k W[rows[r]][k] * x[b][k]        (double accumulation)   */
/*   a[b][r] = sum_k |W[rows[r]][k] * x[b][k]|                              */
/* ------------------------------------------------------------------------ */
int oracle_q4k_gemv_rows(const uint8_t *w, int soa, int64_t N, int64_t K,
                         const float *x, int B, const int64_t *rows, int64_t nrows,
                         double *y, double *a)
{
    if (N < 0 || K < 0 || K % Q4K_BLOCK_ELEMS != 0 || B < 1)
        return -1;
    int64_t nb = K / Q4K_BLOCK_ELEMS;
    uint8_t blk[Q4K_BLOCK_BYTES];
    double wv[Q4K_BLOCK_ELEMS];
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t n = rows[r];
        if (n < 0 || n >= N)
            return -2;
        for (int b = 0; b < B; ++b) {
            y[(int64_t)b * nrows + r] = 0.0;
            a[(int64_t)b * nrows + r] = 0.0;
        }
        const uint8_t *row = w + n * nb * Q4K_BLOCK_BYTES;
        for (int64_t kb = 0; kb < nb; ++kb) {
            gather_q4k_block(row, nb, kb, soa, blk);
            oracle_q4k_block(blk, wv);
            for (int b = 0; b < B; ++b) {
                const float *xb = x + (int64_t)b * K + kb * Q4K_BLOCK_ELEMS;
                double sy = 0.0, sa = 0.0;
                for (int i = 0; i < Q4K_BLOCK_ELEMS; ++i) {
                    double p = wv[i] * (double)xb[i];
                    sy += p;
                    sa += fabs(p);
                }
                y[(int64_t)b * nrows + r] += sy;
                a[(int64_t)b * nrows + r] += sa;
            }
        }
    }
    return 0;
}

int oracle_q8_0_gemv_rows(const uint8_t *w, int64_t N, int64_t K, const float *x, int B,
                          const int64_t *rows, int64_t nrows, double *y, double *a)
{
    if (N < 0 || K < 0 || K % Q8_0_BLOCK_ELEMS != 0 || B < 1)
        return -1;
    int64_t nb = K / Q8_0_BLOCK_ELEMS;
    double wv[Q8_0_BLOCK_ELEMS];
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t n = rows[r];
        if (n < 0 || n >= N)
            return -2;
        for (int b = 0; b < B; ++b) {
            y[(int64_t)b * nrows + r] = 0.0;
            a[(int64_t)b * nrows + r] = 0.0;
        }
        for (int64_t kb = 0; kb < nb; ++kb) {
            oracle_q8_0_block(w + (n * nb + kb) * Q8_0_BLOCK_BYTES, wv);
            for (int b = 0; b < B; ++b) {
                const float *xb = x + (int64_t)b * K + kb * Q8_0_BLOCK_ELEMS;
                for (int i = 0; i < Q8_0_BLOCK_ELEMS; ++i) {
                    double p = wv[i] * (double)xb[i];
                    y[(int64_t)b * nrows + r] += p;
                    a[(int64_t)b * nrows + r] += fabs(p);
                }
            }
        }
    }
    return 0;
}

/* silu(g) * u = g / (1 + e^-g) * u, elementwise, in double. */
void oracle_swiglu(const double *g, const double *u, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = g[i] / (1.0 + exp(-g[i])) * u[i];
}

/* De-interleave of a q-projection-with-gate output (Doppler 0.1.8,
 * split_qg.wgsl).  Each of the B rows of y holds, per head h, head_dim Q values
 * followed by head_dim gate values; Q and G receive them contiguously:
 *   q[b][h*hd + d] = y[b][h*2*hd + d],  g[b][h*hd + d] = y[b][h*2*hd + hd + d].
 * N (the row length of y) must be a positive multiple of 2*hd. */
int oracle_split_qg(const double *y, int64_t B, int64_t N, int64_t hd, double *q, double *g)
{
    if (B < 0 || N <= 0 || hd <= 0 || N % (2 * hd) != 0)
        return -1;
    int64_t qsize = N / 2;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t h = 0; h < N / (2 * hd); ++h)
            for (int64_t d = 0; d < hd; ++d) {
                q[b * qsize + h * hd + d] = y[b * N + h * 2 * hd + d];
                g[b * qsize + h * hd + d] = y[b * N + h * 2 * hd + hd + d];
            }
    return 0;
}

/* Index of the largest value; among equal largest values the lowest index. */
int64_t oracle_argmax(const double *v, int64_t n)
{
    if (n <= 0)
        return -1;
    int64_t best = 0;
    for (int64_t i = 1; i < n; ++i)
        if (v[i] > v[best])
            best = i;
    return best;
}

/* ------------------------------------------------------------------------ */
/* W4A16 prefill: Y = X W^T with 16-bit operands (qualiaDB qwen3_attention: */
/* prefill_weights, "W4A16 M128 dispatcher").  The pages name the operation */
/* and its operand widths only; the reading taken here:                     */
/*   - activations X (M x K) are IEEE binary16 values, given as bit         */
/*     patterns;                                                            */
/*   - each weight is the Q4_K weight rounded once to fp32 (as in           */
/*     oracle_q4k_dequant_f32) and then to binary16, both round to nearest, */
/*     ties to even;                                                        */
/*   - Y (M x N) is the exact sum of those products (every product of two   */
/*     binary16 values is exact in double; the double sum is the oracle).   */
/* ------------------------------------------------------------------------ */

/* fp32 -> IEEE binary16 bit pattern, round to nearest, ties to even.
 * binary16 has an 11-bit significand; normal values are m * 2^(E-10) with
 * 1024 <= m < 2048 and -14 <= E <= 15, subnormals m * 2^-24 with m < 1024.
 * |f| >= 65520 (half-way between the largest finite value 65504 and 2^16)
 * rounds to infinity.  NaN gives the quiet NaN 0x7E00 with f's sign. */
uint16_t oracle_float_to_fp16(float f)
{
    double v = (double)f;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (isnan(v))
        return (uint16_t)(sign | 0x7E00);
    if (a >= 65520.0)
        return (uint16_t)(sign | 0x7C00);
    if (a < ldexp(1.0, -14)) {
        /* subnormal (or zero): m = a / 2^-24 rounded; m == 1024 is 2^-14 */
        double m = nearbyint(ldexp(a, 24));
        return (uint16_t)(sign | (uint16_t)m);
    }
    int ex;
    frexp(a, &ex);              /* a = fr * 2^ex, 0.5 <= fr < 1 */
    int E = ex - 1;             /* 2^E <= a < 2^(E+1) */
    double m = nearbyint(ldexp(a, 10 - E));   /* in [1024, 2048] */
    if (m == 2048.0) {
        m = 1024.0;
        E += 1;
    }
    /* E <= 15 here: a < 65520 rounds to at most 65504 = 2047 * 2^5 */
    return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | (uint16_t)(m - 1024.0));
}

void oracle_float_to_fp16_array(const float *f, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_float_to_fp16(f[i]);
}

/* Q4_K matrix -> binary16 weights (N x K bit patterns), as defined above. */
int oracle_q4k_dequant_f16(const uint8_t *w, int soa, int64_t N, int64_t K, uint16_t *out)
{
    if (N < 0 || K < 0 || K % Q4K_BLOCK_ELEMS != 0)
        return -1;
    int64_t nb = K / Q4K_BLOCK_ELEMS;
    uint8_t blk[Q4K_BLOCK_BYTES];
    double tmp[Q4K_BLOCK_ELEMS];
    for (int64_t n = 0; n < N; ++n) {
        const uint8_t *row = w + n * nb * Q4K_BLOCK_BYTES;
        for (int64_t kb = 0; kb < nb; ++kb) {
            gather_q4k_block(row, nb, kb, soa, blk);
            oracle_q4k_block(blk, tmp);
            for (int i = 0; i < Q4K_BLOCK_ELEMS; ++i)
                out[n * K + kb * Q4K_BLOCK_ELEMS + i] = oracle_float_to_fp16((float)tmp[i]);
        }
    }
    return 0;
}

/* Prefill product on a list of weight rows.  x16 is M x K binary16 bit
 * patterns (row-major); y and a are M x nrows (row-major):
 *   y[m][r] = sum_k W16[rows[r]][k] * X16[m][k]      (double accumulation)
 *   a[m][r] = sum_k |W16[rows[r]][k] * X16[m][k]|                           */
int oracle_q4k_prefill_rows(const uint8_t *w, int soa, int64_t N, int64_t K,
                            const uint16_t *x16, int64_t M, const int64_t *rows, int64_t nrows,
                            double *y, double *a)
{
    if (N < 0 || K < 0 || K % Q4K_BLOCK_ELEMS != 0 || M < 1)
        return -1;
    int64_t nb = K / Q4K_BLOCK_ELEMS;
    uint8_t blk[Q4K_BLOCK_BYTES];
    double wv[Q4K_BLOCK_ELEMS];
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t n = rows[r];
        if (n < 0 || n >= N)
            return -2;
        for (int64_t m = 0; m < M; ++m) {
            y[m * nrows + r] = 0.0;
            a[m * nrows + r] = 0.0;
        }
        const uint8_t *row = w + n * nb * Q4K_BLOCK_BYTES;
        for (int64_t kb = 0; kb < nb; ++kb) {
            gather_q4k_block(row, nb, kb, soa, blk);
            oracle_q4k_block(blk, wv);
            for (int i = 0; i < Q4K_BLOCK_ELEMS; ++i)
                wv[i] = oracle_fp16_to_double(oracle_float_to_fp16((float)wv[i]));
            for (int64_t m = 0; m < M; ++m) {
                const uint16_t *xm = x16 + m * K + kb * Q4K_BLOCK_ELEMS;
                double sy = 0.0, sa = 0.0;
                for (int i = 0; i < Q4K_BLOCK_ELEMS; ++i) {
                    double p = wv[i] * oracle_fp16_to_double(xm[i]);
                    sy += p;
                    sa += fabs(p);
                }
                y[m * nrows + r] += sy;
                a[m * nrows + r] += sa;
            }
        }
    }
    return 0;
}
