/*
 * oracle.c - plain CPU reference for the MoE low-precision quantization path.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's CPU
 * baseline leg may load this library. It is single threaded, deliberately slow
 * and written straight from the definitions; it shares no source, header,
 * table or helper with the CUDA library, and the CUDA library never calls it.
 *
 * Sources (pytorch/ao pull-request pages; cited by number, title and section):
 *   #2064 "[scaled grouped mm] add triton kernels for float8 rowwise
 *         quantization with per-group/jagged scales"  - Motivation, Summary
 *   #2827 "[fp8 blockwise] load 2d chunks for groupwise quant to enable
 *         coalesced gmem accesses"                     - description
 *   #3002 "[mxfp8 moe training] add CUDA kernel to quantize 3d tensor colwise"
 *                                                      - Summary, comments
 *   #3504 "[mxfp8 moe training] add CUDA kernel for per-group conversion of
 *         scale factors to blocked layout"             - title, Benchmarks
 * plus the definitions those pages rely on but do not print:
 *   - float8 e4m3 ("E4M3FN"): 1 sign, 4 exponent (bias 7), 3 mantissa bits,
 *     no infinities, 0x7F/0xFF are NaN, largest finite value 448;
 *   - OCP Microscaling (MX) v1.0: E8M0 shared scale, element emax 8 for e4m3;
 *   - the 128x4 "blocked" scale-factor layout consumed by block-scaled GEMMs.
 *
 * Readings taken where the pages are silent (each one is listed, with its
 * reason, in the design notes of the repository):
 *   R1 e4m3 scale s = fp32(448 / max(amax, fp32(1e-12))); the stored scale is
 *      the fp32 reciprocal fp32(1 / s).
 *   R2 cast = clamp to [-448, 448] then round-to-nearest-even; sign of zero kept.
 *   R3 offsets are int32 cumulative group ends; group g = [end[g-1], end[g]).
 *   R4 empty groups and all-zero units still get a scale (amax clamps to 1e-12).
 *   R5 MX floor:  scale exponent = floor(log2 amax) - 8, clamped to [-127,127].
 *      MX rceil:  scale exponent = ceil(log2(amax / 448)), clamped likewise.
 *      amax == 0 gives the smallest scale, byte 0.
 *   R6 MX element = cast(x / 2^(byte-127)), an exact power-of-two division.
 *   R7 scale layouts: jagged (G, lines); blockwise (rows/br, cols/bc);
 *      MX 3-D (E, K, N/32); MX rowwise (rows, cols/32); all row-major.
 *   R8 blocked layout: pad rows to 128 and cols to 4 with zero bytes, then each
 *      128x4 tile is stored as (32, 4, 4): byte (r, c) of the tile goes to
 *      (r % 32) * 16 + (r / 32) * 4 + c; tiles are ordered row-tile major.
 *   R9 grouped blocked layout: each group's rows are padded to a multiple of
 *      128 on their own; groups are stacked in order; the rest is zero.
 *   R12 groups along K (#3504's stack, #3505): each group's scale columns are
 *      padded to a multiple of 4 on their own and placed side by side in one
 *      matrix of 128-padded rows and capacity_cols columns, which is stored
 *      in the blocked layout of R8; the rest is zero (the pages' byte count,
 *      R*C read and R*(C + 4G) written, fits this single output matrix).
 *   R13 MX rowwise quantization with blocked scales = the rowwise op followed
 *      by the row-group conversion of R9 applied to its scales.
 *
 * Floating point: every step the definitions place in fp32 is done in fp32
 * (C float arithmetic, round-to-nearest, no contraction, no flush to zero);
 * exact steps (power-of-two scaling, e4m3 rounding decisions) are done in
 * double where the values are exactly representable.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "oracle.h"

/* ------------------------------------------------------------------ */
/* scalar definitions                                                  */
/* ------------------------------------------------------------------ */

/* bfloat16 is the upper half of an IEEE binary32 word. */
static float bf16_value(uint16_t bits)
{
    uint32_t w = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return f;
}

/* Value of an e4m3 code, straight from the field definition. */
double oracle_e4m3_value(uint8_t code)
{
    unsigned sign = code >> 7;
    unsigned expo = (code >> 3) & 0xF;
    unsigned mant = code & 0x7;
    double mag;
    if (expo == 0xF && mant == 0x7)
        return NAN;
    if (expo == 0)
        mag = ldexp((double)mant, -9);               /* m/8 * 2^(1-7) */
    else
        mag = ldexp((double)(8 + mant), (int)expo - 10); /* (1+m/8) * 2^(e-7) */
    return sign ? -mag : mag;
}

/* fp32 -> e4m3: clamp to [-448, 448], then round to the nearest code, ties to
 * the code whose last mantissa bit is 0. The non-negative finite codes 0..126
 * are ordered by value, so a binary search finds the two neighbours; their
 * midpoint has at most five significant bits and is exact in double, so the
 * comparison with the (exact) input is exact. */
uint8_t oracle_e4m3_from_float(float v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    unsigned lo, hi;
    double below, above, mid;
    if (isnan(v))
        return (uint8_t)(sign | 0x7F); /* outside the contract */
    if (a >= 448.0)
        return (uint8_t)(sign | 0x7E);
    lo = 0;
    hi = 126;
    while (lo < hi) { /* largest code with value <= a */
        unsigned m = (lo + hi + 1) / 2;
        if (oracle_e4m3_value((uint8_t)m) <= a)
            lo = m;
        else
            hi = m - 1;
    }
    below = oracle_e4m3_value((uint8_t)lo);
    above = oracle_e4m3_value((uint8_t)(lo + 1));
    mid = 0.5 * (below + above);
    if (a < mid)
        return (uint8_t)(sign | lo);
    if (a > mid)
        return (uint8_t)(sign | (lo + 1));
    return (uint8_t)(sign | ((lo & 1) ? lo + 1 : lo));
}

void oracle_e4m3_from_float_array(const float *v, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_e4m3_from_float(v[i]);
}

/* R1: the per-unit e4m3 scale, in fp32 (#2064 Summary: dynamic float8
 * quantization with one scale per row / column of each group). */
float oracle_fp8_scale(float amax)
{
    const float eps = 1e-12f;
    float d = amax > eps ? amax : eps;
    return 448.0f / d;
}

float oracle_fp8_inv_scale(float amax)
{
    return 1.0f / oracle_fp8_scale(amax);
}

static uint8_t clamp_e8m0(int k)
{
    if (k < -127)
        k = -127;
    if (k > 127)
        k = 127;
    return (uint8_t)(k + 127);
}

/* R5 floor: OCP MX v1.0 shared exponent floor(log2 amax) - emax(e4m3 = 8).
 * ilogb on the exact double value is floor(log2) for every positive input,
 * fp32 subnormals included. */
uint8_t oracle_e8m0_floor(float amax)
{
    if (!(amax > 0.0f))
        return 0;
    return clamp_e8m0(ilogb((double)amax) - 8);
}

/* R5 rceil (#3002 comments name the "floor, rceil" scale modes): the smallest
 * power of two X with amax / X <= 448, i.e. k = ceil(log2(amax / 448)).
 * 448 * 2^k is exact in double over the whole range, so both loops compare
 * exactly; on exit 448*2^k >= amax and 448*2^(k-1) < amax. */
uint8_t oracle_e8m0_rceil(float amax)
{
    double a = (double)amax;
    int k;
    if (!(amax > 0.0f))
        return 0;
    k = ilogb(a) - 8;
    while (ldexp(448.0, k) < a)
        ++k;
    while (ldexp(448.0, k - 1) >= a)
        --k;
    return clamp_e8m0(k);
}

uint8_t oracle_e8m0(float amax, int mode)
{
    return mode == ORACLE_RCEIL ? oracle_e8m0_rceil(amax) : oracle_e8m0_floor(amax);
}

/* R6: element = cast(x / 2^(byte-127)). The quotient is exact in double and
 * the conversion to float is the single fp32 rounding. */
uint8_t oracle_mx_element(float x, uint8_t scale_byte)
{
    double q = (double)x / ldexp(1.0, (int)scale_byte - 127);
    return oracle_e4m3_from_float((float)q);
}

/* R8: byte offset of element (r, c) of a row-major matrix with padded column
 * count cols_padded (a multiple of 4) inside its 128x4 blocked layout. */
int64_t oracle_blocked_offset(int64_t r, int64_t c, int64_t cols_padded)
{
    int64_t tile = (r / 128) * (cols_padded / 4) + c / 4;
    int64_t rr = r % 128;
    return tile * 512 + (rr % 32) * 16 + (rr / 32) * 4 + (c % 4);
}

/* ------------------------------------------------------------------ */
/* helpers                                                             */
/* ------------------------------------------------------------------ */

/* R3: int32 cumulative ends, non-decreasing, within [0, extent]. */
static int offsets_valid(const int32_t *offs, int32_t groups, int64_t extent)
{
    int64_t prev = 0;
    for (int32_t g = 0; g < groups; ++g) {
        if (offs[g] < prev || offs[g] > extent)
            return 0;
        prev = offs[g];
    }
    return 1;
}

static float absf(float x) { return x < 0.0f ? -x : (x > 0.0f ? x : 0.0f); }

/* ------------------------------------------------------------------ */
/* (a1) jagged rowwise: one scale per (row, group), groups are column   */
/* ranges; row-major output. #2064 Summary, first kernel.              */
/* ------------------------------------------------------------------ */
int oracle_fp8_quant_jagged_rowwise(const uint16_t *in, int64_t rows, int64_t cols,
                                    int64_t stride_row, int64_t stride_col,
                                    const int32_t *offs, int32_t groups,
                                    uint8_t *out, float *inv_scales)
{
    if (rows < 0 || cols < 0 || groups <= 0)
        return ORACLE_ERR_ARG;
    if (!offsets_valid(offs, groups, cols))
        return ORACLE_ERR_OFFSETS;
    for (int64_t r = 0; r < rows; ++r) {
        int64_t start = 0;
        for (int32_t g = 0; g < groups; ++g) {
            int64_t end = offs[g];
            float amax = 0.0f, s;
            for (int64_t c = start; c < end; ++c) {
                float a = absf(bf16_value(in[r * stride_row + c * stride_col]));
                if (a > amax)
                    amax = a;
            }
            s = oracle_fp8_scale(amax);
            inv_scales[(int64_t)g * rows + r] = 1.0f / s;
            for (int64_t c = start; c < end; ++c) {
                float y = bf16_value(in[r * stride_row + c * stride_col]) * s;
                out[r * cols + c] = oracle_e4m3_from_float(y);
            }
            start = end;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* (a2) jagged colwise: one scale per (column, group), groups are row   */
/* ranges; column-major output out[c * rows + r]. #2064 Summary.       */
/* ------------------------------------------------------------------ */
int oracle_fp8_quant_jagged_colwise(const uint16_t *in, int64_t rows, int64_t cols,
                                    int64_t stride_row, int64_t stride_col,
                                    const int32_t *offs, int32_t groups,
                                    uint8_t *out, float *inv_scales)
{
    if (rows < 0 || cols < 0 || groups <= 0)
        return ORACLE_ERR_ARG;
    if (!offsets_valid(offs, groups, rows))
        return ORACLE_ERR_OFFSETS;
    for (int64_t c = 0; c < cols; ++c) {
        int64_t start = 0;
        for (int32_t g = 0; g < groups; ++g) {
            int64_t end = offs[g];
            float amax = 0.0f, s;
            for (int64_t r = start; r < end; ++r) {
                float a = absf(bf16_value(in[r * stride_row + c * stride_col]));
                if (a > amax)
                    amax = a;
            }
            s = oracle_fp8_scale(amax);
            inv_scales[(int64_t)g * cols + c] = 1.0f / s;
            for (int64_t r = start; r < end; ++r) {
                float y = bf16_value(in[r * stride_row + c * stride_col]) * s;
                out[c * rows + r] = oracle_e4m3_from_float(y);
            }
            start = end;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* (a3) blockwise: one scale per br x bc block of a row-major matrix    */
/* (1x128 activations, 128x128 weights). #2827 description.            */
/* ------------------------------------------------------------------ */
int oracle_fp8_quant_blockwise(const uint16_t *in, int64_t rows, int64_t cols,
                               int32_t br, int32_t bc, uint8_t *out, float *inv_scales)
{
    int64_t nbr, nbc;
    if (rows < 0 || cols < 0 || br <= 0 || bc <= 0 || rows % br || cols % bc)
        return ORACLE_ERR_ARG;
    nbr = rows / br;
    nbc = cols / bc;
    for (int64_t bi = 0; bi < nbr; ++bi) {
        for (int64_t bj = 0; bj < nbc; ++bj) {
            float amax = 0.0f, s;
            for (int64_t r = bi * br; r < (bi + 1) * br; ++r)
                for (int64_t c = bj * bc; c < (bj + 1) * bc; ++c) {
                    float a = absf(bf16_value(in[r * cols + c]));
                    if (a > amax)
                        amax = a;
                }
            s = oracle_fp8_scale(amax);
            inv_scales[bi * nbc + bj] = 1.0f / s;
            for (int64_t r = bi * br; r < (bi + 1) * br; ++r)
                for (int64_t c = bj * bc; c < (bj + 1) * bc; ++c)
                    out[r * cols + c] = oracle_e4m3_from_float(bf16_value(in[r * cols + c]) * s);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Blockwise with transposed output (#2827 description: the (blocksize */
/* x 1) tiles of the blockwise linear, and the transposed weight). The  */
/* row-major (rows, cols) input is quantized in br x bc blocks          */
/* (br = 128; bc = 1 or 128) and written transposed: out[c*rows + r],   */
/* one inverse scale per block at inv[(c/bc) * (rows/br) + r/br], i.e.  */
/* the (cols/bc, rows/br) row-major scale matrix of the transpose.      */
/* ------------------------------------------------------------------ */
int oracle_fp8_quant_blockwise_transposed(const uint16_t *in, int64_t rows, int64_t cols,
                                          int32_t br, int32_t bc, uint8_t *out, float *inv_scales)
{
    int64_t nbr, nbc;
    if (rows < 0 || cols < 0 || br <= 0 || bc <= 0 || rows % br || cols % bc)
        return ORACLE_ERR_ARG;
    nbr = rows / br;
    nbc = cols / bc;
    for (int64_t bj = 0; bj < nbc; ++bj) {
        for (int64_t bi = 0; bi < nbr; ++bi) {
            float amax = 0.0f, s;
            for (int64_t r = bi * br; r < (bi + 1) * br; ++r)
                for (int64_t c = bj * bc; c < (bj + 1) * bc; ++c) {
                    float a = absf(bf16_value(in[r * cols + c]));
                    if (a > amax)
                        amax = a;
                }
            s = oracle_fp8_scale(amax);
            inv_scales[bj * nbr + bi] = 1.0f / s;
            for (int64_t r = bi * br; r < (bi + 1) * br; ++r)
                for (int64_t c = bj * bc; c < (bj + 1) * bc; ++c)
                    out[c * rows + r] = oracle_e4m3_from_float(bf16_value(in[r * cols + c]) * s);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* (a4) MX 3-D colwise: expert weights (E, N, K) quantized along N in   */
/* 32x1 blocks, each expert written column-major:                       */
/* out[e*N*K + k*N + n], scales (E, K, N/32). #3002 Summary.            */
/* ------------------------------------------------------------------ */
int oracle_mx_quant_3d_colwise(const uint16_t *in, int64_t E, int64_t N, int64_t K,
                               int mode, uint8_t *out, uint8_t *scales)
{
    if (E < 0 || N < 0 || K < 0 || N % 32)
        return ORACLE_ERR_ARG;
    for (int64_t e = 0; e < E; ++e) {
        const uint16_t *w = in + e * N * K;
        for (int64_t k = 0; k < K; ++k) {
            for (int64_t b = 0; b < N / 32; ++b) {
                float amax = 0.0f;
                uint8_t byte;
                for (int64_t n = b * 32; n < b * 32 + 32; ++n) {
                    float a = absf(bf16_value(w[n * K + k]));
                    if (a > amax)
                        amax = a;
                }
                byte = oracle_e8m0(amax, mode);
                scales[(e * K + k) * (N / 32) + b] = byte;
                for (int64_t n = b * 32; n < b * 32 + 32; ++n)
                    out[e * N * K + k * N + n] = oracle_mx_element(bf16_value(w[n * K + k]), byte);
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* (a5) MX rowwise: 1x32 blocks along the last dimension; row-major     */
/* output and scales (rows, cols/32). The last-dim scaling that #3002   */
/* Summary attributes to to_mx.                                         */
/* ------------------------------------------------------------------ */
int oracle_mx_quant_rowwise(const uint16_t *in, int64_t rows, int64_t cols, int mode,
                            uint8_t *out, uint8_t *scales)
{
    if (rows < 0 || cols < 0 || cols % 32)
        return ORACLE_ERR_ARG;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < cols / 32; ++b) {
            float amax = 0.0f;
            uint8_t byte;
            for (int64_t c = b * 32; c < b * 32 + 32; ++c) {
                float a = absf(bf16_value(in[r * cols + c]));
                if (a > amax)
                    amax = a;
            }
            byte = oracle_e8m0(amax, mode);
            scales[r * (cols / 32) + b] = byte;
            for (int64_t c = b * 32; c < b * 32 + 32; ++c)
                out[r * cols + c] = oracle_mx_element(bf16_value(in[r * cols + c]), byte);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* (a6) per-group conversion of a (rows, cols) scale matrix to the      */
/* blocked layout, each group's rows padded to 128 on their own (#3504  */
/* title). Output: capacity_rows x pad4(cols) bytes, every byte set.    */
/* ------------------------------------------------------------------ */
int64_t oracle_blocked_grouped_rows_bound(int64_t rows, int32_t groups)
{
    /* sum_g 128*ceil(s_g/128) <= 128*floor((rows + 127*groups) / 128) */
    return 128 * ((rows + 127 * (int64_t)groups) / 128);
}

int oracle_mx_scales_to_blocked_grouped(const uint8_t *scales, int64_t rows, int64_t cols,
                                        const int32_t *offs, int32_t groups,
                                        uint8_t *out, int64_t capacity_rows,
                                        int32_t *group_row_starts)
{
    int64_t cols_p, start = 0, base = 0;
    if (rows < 0 || cols < 0 || groups <= 0 || capacity_rows < 0)
        return ORACLE_ERR_ARG;
    if (capacity_rows % 128 || capacity_rows < oracle_blocked_grouped_rows_bound(rows, groups))
        return ORACLE_ERR_ARG;
    if (!offsets_valid(offs, groups, rows))
        return ORACLE_ERR_OFFSETS;
    cols_p = (cols + 3) / 4 * 4;
    memset(out, 0, (size_t)(capacity_rows * cols_p));
    for (int32_t g = 0; g < groups; ++g) {
        int64_t end = offs[g], size = end - start;
        if (group_row_starts)
            group_row_starts[g] = (int32_t)base;
        for (int64_t r = 0; r < size; ++r)
            for (int64_t c = 0; c < cols; ++c)
                out[oracle_blocked_offset(base + r, c, cols_p)] = scales[(start + r) * cols + c];
        base += (size + 127) / 128 * 128;
        start = end;
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Groups along K (ao PR 3504's stack, #3505 "integrate new cuda kernel */
/* for blocked layout for groups along K"). Group g is the scale-column */
/* range [offs[g-1], offs[g]). Reading taken where the pages are        */
/* silent (their byte count, R*C in and R*(C + 4G) out, fits one output */
/* matrix): each group's columns are padded to a multiple of 4 on their */
/* own and placed side by side from column Q_g = sum_{h<g}              */
/* 4*ceil(size_h/4); rows are padded to a multiple of 128; the whole    */
/* (128*ceil(rows/128), capacity_cols) matrix is stored in the 128x4    */
/* blocked layout, every byte not taken by a scale being zero.          */
/* ------------------------------------------------------------------ */
int64_t oracle_blocked_grouped_k_cols_bound(int64_t cols, int32_t groups)
{
    /* sum_g 4*ceil(s_g/4) is a multiple of 4 and at most cols + 3*groups */
    return 4 * ((cols + 3 * (int64_t)groups) / 4);
}

int oracle_mx_scales_to_blocked_grouped_k(const uint8_t *scales, int64_t rows, int64_t cols,
                                          const int32_t *offs, int32_t groups,
                                          uint8_t *out, int64_t capacity_cols,
                                          int32_t *group_col_starts)
{
    int64_t rows_p, start = 0, base = 0;
    if (rows < 0 || cols < 0 || groups <= 0 || capacity_cols < 0)
        return ORACLE_ERR_ARG;
    if (capacity_cols % 4 || capacity_cols < oracle_blocked_grouped_k_cols_bound(cols, groups))
        return ORACLE_ERR_ARG;
    if (!offsets_valid(offs, groups, cols))
        return ORACLE_ERR_OFFSETS;
    rows_p = (rows + 127) / 128 * 128;
    memset(out, 0, (size_t)(rows_p * capacity_cols));
    for (int32_t g = 0; g < groups; ++g) {
        int64_t end = offs[g], size = end - start;
        if (group_col_starts)
            group_col_starts[g] = (int32_t)base;
        for (int64_t r = 0; r < rows; ++r)
            for (int64_t c = 0; c < size; ++c)
                out[oracle_blocked_offset(r, base + c, capacity_cols)] = scales[r * cols + start + c];
        base += (size + 3) / 4 * 4;
        start = end;
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* MX rowwise quantization whose E8M0 scales go straight to the         */
/* per-group blocked layout: by definition the rowwise op (a5) followed */
/* by the row-group conversion (a6) of its scales.                     */
/* ------------------------------------------------------------------ */
int oracle_mx_quant_rowwise_blocked_grouped(const uint16_t *in, int64_t rows, int64_t cols, int mode,
                                            const int32_t *offs, int32_t groups,
                                            uint8_t *out, uint8_t *scales_blocked,
                                            int64_t capacity_rows, int32_t *group_row_starts)
{
    uint8_t *scales;
    int rc;
    if (rows < 0 || cols < 0 || cols % 32)
        return ORACLE_ERR_ARG;
    scales = (uint8_t *)malloc((size_t)(rows * (cols / 32)) + 1);
    if (!scales)
        return ORACLE_ERR_ARG;
    rc = oracle_mx_quant_rowwise(in, rows, cols, mode, out, scales);
    if (rc == 0)
        rc = oracle_mx_scales_to_blocked_grouped(scales, rows, cols / 32, offs, groups, scales_blocked,
                                                 capacity_rows, group_row_starts);
    free(scales);
    return rc;
}

/* ------------------------------------------------------------------ */
/* FP8 rowwise-scaled grouped GEMM, the consumer of these buffers       */
/* (#2064 Motivation and #2077 Summary: the differentiable scaled       */
/* grouped mm the quantization feeds). Row m of A belongs to the group  */
/* g with offs[g-1] <= m < offs[g]; its output row is                    */
/*   out[m][n] = (sum_k e4m3(a[m][k]) * e4m3(w[g][n][k])) * inv_a[m]     */
/*               * inv_w[g][n]                                           */
/* computed in double (every e4m3 product is exact in double; the sum of */
/* K of them is exact to far below fp32 resolution). Rows past          */
/* offs[G-1] are not written.                                            */
/* ------------------------------------------------------------------ */
int oracle_fp8_grouped_gemm_rowwise(const uint8_t *a, const float *inv_a, const uint8_t *w, const float *inv_w,
                                    int64_t M, int64_t N, int64_t K, const int32_t *offs, int32_t groups,
                                    double *out)
{
    int64_t start = 0;
    if (M < 0 || N < 0 || K < 0 || groups <= 0)
        return ORACLE_ERR_ARG;
    if (!offsets_valid(offs, groups, M))
        return ORACLE_ERR_OFFSETS;
    for (int32_t g = 0; g < groups; ++g) {
        const uint8_t *wg = w + (int64_t)g * N * K;
        for (int64_t m = start; m < offs[g]; ++m) {
            for (int64_t n = 0; n < N; ++n) {
                double acc = 0.0;
                for (int64_t k = 0; k < K; ++k)
                    acc += oracle_e4m3_value(a[m * K + k]) * oracle_e4m3_value(wg[n * K + k]);
                out[m * N + n] = acc * (double)inv_a[m] * (double)inv_w[(int64_t)g * N + n];
            }
        }
        start = offs[g];
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* MXFP8 block-scaled grouped GEMM, the consumer of the MX rowwise      */
/* quantization and of the blocked scale layout (#3504 title: blocked   */
/* scales per group for MXFP8 MoE training; reading R18: they feed the  */
/* MoE layer's grouped GEMM). By the OCP MX definition an element's     */
/* value is its e4m3 value times 2^(e - 127)                            */
/* of its block's E8M0 byte e (255 is NaN), blocks being 32 consecutive */
/* elements along K. Row m of group g:                                  */
/*   out[m][n] = sum_k x(a[m][k], sa[m][k/32]) * x(w[g][n][k], sw[g][n][k/32]) */
/* with x(c, e) = e4m3(c) * 2^(e-127); the scales are passed in their    */
/* plain row-major layouts, sa (M, K/32) and sw (G, N, K/32). In double */
/* (each product is exact; the sum of K of them is exact far below fp32 */
/* resolution). Rows past offs[G-1] are not written.                     */
/* ------------------------------------------------------------------ */
static double e8m0_value(uint8_t e)
{
    return e == 255 ? NAN : ldexp(1.0, (int)e - 127);
}

int oracle_mx_grouped_gemm(const uint8_t *a, const uint8_t *sa, const uint8_t *w, const uint8_t *sw,
                           int64_t M, int64_t N, int64_t K, const int32_t *offs, int32_t groups, double *out)
{
    int64_t start = 0, kb = K / 32;
    if (M < 0 || N < 0 || K < 0 || K % 32 || groups <= 0)
        return ORACLE_ERR_ARG;
    if (!offsets_valid(offs, groups, M))
        return ORACLE_ERR_OFFSETS;
    for (int32_t g = 0; g < groups; ++g) {
        const uint8_t *wg = w + (int64_t)g * N * K, *swg = sw + (int64_t)g * N * kb;
        for (int64_t m = start; m < offs[g]; ++m) {
            for (int64_t n = 0; n < N; ++n) {
                double acc = 0.0;
                for (int64_t k = 0; k < K; ++k)
                    acc += oracle_e4m3_value(a[m * K + k]) * e8m0_value(sa[m * kb + k / 32]) *
                           (oracle_e4m3_value(wg[n * K + k]) * e8m0_value(swg[n * kb + k / 32]));
                out[m * N + n] = acc;
            }
        }
        start = offs[g];
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* MX quantization along the grouped dimension, for the weight gradient */
/* of the MXFP8 grouped GEMM (reading R19: #3505 "integrate new cuda    */
/* kernel for blocked layout for groups along K" implies scales grouped */
/* along the contracted token dimension; here each group's tokens are   */
/* cut into 32-element MX blocks starting at the group's first token,   */
/* the last block of a group holding the remainder). Element (r, c) of  */
/* a (rows, cols) bf16 matrix with rows grouped by offs; per column c   */
/* and block j of group g (rows s_g + 32j .. min(s_g + 32j + 32, e_g)): */
/* byte = E8M0(amax over the block) by `mode`, out[c * rows + r] =      */
/* mx_element(x, byte) (column-major), scales[c * nblk + B_g + j] with  */
/* B_g = sum_{h<g} ceil(size_h / 32) and nblk = B_G. Rows past          */
/* offs[G-1] are not written.                                            */
/* ------------------------------------------------------------------ */
int64_t oracle_mx_jagged_blocks(const int32_t *offs, int32_t groups)
{
    int64_t n = 0, start = 0;
    for (int32_t g = 0; g < groups; ++g) {
        n += (offs[g] - start + 31) / 32;
        start = offs[g];
    }
    return n;
}

int oracle_mx_quant_jagged_colwise(const uint16_t *in, int64_t rows, int64_t cols, int64_t stride_row,
                                   int64_t stride_col, const int32_t *offs, int32_t groups, int mode, uint8_t *out,
                                   uint8_t *scales)
{
    int64_t nblk;
    if (rows < 0 || cols < 0 || groups <= 0)
        return ORACLE_ERR_ARG;
    if (!offsets_valid(offs, groups, rows))
        return ORACLE_ERR_OFFSETS;
    nblk = oracle_mx_jagged_blocks(offs, groups);
    for (int64_t c = 0; c < cols; ++c) {
        int64_t start = 0, base = 0;
        for (int32_t g = 0; g < groups; ++g) {
            const int64_t end = offs[g];
            for (int64_t j = 0; start + 32 * j < end; ++j) {
                const int64_t r0 = start + 32 * j, r1 = r0 + 32 < end ? r0 + 32 : end;
                float amax = 0.0f;
                uint8_t byte;
                for (int64_t r = r0; r < r1; ++r) {
                    float a = absf(bf16_value(in[r * stride_row + c * stride_col]));
                    if (a > amax)
                        amax = a;
                }
                byte = oracle_e8m0(amax, mode);
                scales[c * nblk + base + j] = byte;
                for (int64_t r = r0; r < r1; ++r)
                    out[c * rows + r] = oracle_mx_element(bf16_value(in[r * stride_row + c * stride_col]), byte);
            }
            base += (end - start + 31) / 32;
            start = end;
        }
    }
    return 0;
}

/* The MXFP8 weight-gradient product over each group's tokens (R19):    */
/*   out[g][n][k] = sum_{m in group g} x(a[n][m], sa[n][B_g + (m-s_g)/32]) */
/*                                    * x(b[k][m], sb[k][B_g + (m-s_g)/32]) */
/* with x(c, e) = e4m3(c) * 2^(e-127); a (N, M) and b (K, M) keep M      */
/* contiguous (the column-major buffers above, of grad_out and of the    */
/* input), sa (N, nblk) and sb (K, nblk). Empty groups give zeros. In    */
/* double.                                                                */
int oracle_mx_grouped_gemm_wgrad(const uint8_t *a, const uint8_t *sa, const uint8_t *b, const uint8_t *sb,
                                 int64_t N, int64_t K, int64_t M, const int32_t *offs, int32_t groups, double *out)
{
    int64_t start = 0, base = 0, nblk;
    if (N < 0 || K < 0 || M < 0 || groups <= 0)
        return ORACLE_ERR_ARG;
    if (!offsets_valid(offs, groups, M))
        return ORACLE_ERR_OFFSETS;
    nblk = oracle_mx_jagged_blocks(offs, groups);
    for (int32_t g = 0; g < groups; ++g) {
        const int64_t end = offs[g];
        for (int64_t n = 0; n < N; ++n)
            for (int64_t k = 0; k < K; ++k) {
                double acc = 0.0;
                for (int64_t m = start; m < end; ++m) {
                    const int64_t j = base + (m - start) / 32;
                    acc += oracle_e4m3_value(a[n * M + m]) * e8m0_value(sa[n * nblk + j]) *
                           (oracle_e4m3_value(b[k * M + m]) * e8m0_value(sb[k * nblk + j]));
                }
                out[((int64_t)g * N + n) * K + k] = acc;
            }
        base += (end - start + 31) / 32;
        start = end;
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Weight-gradient grouped GEMM, the backward consumer of the jagged    */
/* ops (#2064 Summary: the per-group scaled operands of the grad_weight */
/* grouped GEMM). The contraction runs over each group's own positions: */
/*   out[g][n][k] = (sum_{m in group g} e4m3(a[n][m]) * e4m3(b[k][m]))   */
/*                  * inv_a[g][n] * inv_b[g][k]                          */
/* with a (N, M) = grad_out^T quantized rowwise per (row, group) and    */
/* b (K, M) = the input quantized colwise per (column, group), both     */
/* stored with M contiguous. Empty groups give zeros. In double.        */
/* ------------------------------------------------------------------ */
int oracle_fp8_grouped_gemm_wgrad(const uint8_t *a, const float *inv_a, const uint8_t *b, const float *inv_b,
                                  int64_t N, int64_t K, int64_t M, const int32_t *offs, int32_t groups,
                                  double *out)
{
    int64_t start = 0;
    if (M < 0 || N < 0 || K < 0 || groups <= 0)
        return ORACLE_ERR_ARG;
    if (!offsets_valid(offs, groups, M))
        return ORACLE_ERR_OFFSETS;
    for (int32_t g = 0; g < groups; ++g) {
        for (int64_t n = 0; n < N; ++n) {
            for (int64_t k = 0; k < K; ++k) {
                double acc = 0.0;
                for (int64_t m = start; m < offs[g]; ++m)
                    acc += oracle_e4m3_value(a[n * M + m]) * oracle_e4m3_value(b[k * M + m]);
                out[((int64_t)g * N + n) * K + k] =
                    acc * (double)inv_a[(int64_t)g * N + n] * (double)inv_b[(int64_t)g * K + k];
            }
        }
        start = offs[g];
    }
    return 0;
}

