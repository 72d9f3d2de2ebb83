/*
 * fp4_oracle.c — plain CPU oracle for microscaling FP4 (MXFP4 / NVFP4),
 * the block-diagonal Hadamard rotation and the W4A4 product.
 *
 * TEST INFRASTRUCTURE ONLY: used by tests/, the smoke check and the CPU
 * baseline of the benchmark.  The product path never links it.  It is
 * deliberately slow and written step by step in the order the method is
 * described; no blocking, vectorisation or reordering beyond that.
 *
 * Sources (web pages; section / equation / table):
 *   [TransFP4]  "Portable FP4 quantization (TransFP4)", elexvx.com research:
 *               §1.1 Eq.(1) microscaling form; §2.3 Eq.(2) orthogonal
 *               rotation; §3.1 absmax scale + nearest rounding; §3.2 NMSE.
 *   [Guide]     "4.5 FP8 and NVFP4/MXFP4" (inference guide): §1.1 E4M3 bit
 *               pattern 00111000 = 1.0; §1.2 E4M3 max 448, spacing; §3.1 the
 *               E2M1 magnitudes {0,0.5,1,1.5,2,3,4,6}; §3.3 scale formats;
 *               §4.1 NVFP4 two-level dequantization s_tensor*s_block*q.
 *   [Explainer] "MXFP4 quantization explainer" (AI Daily 2026-08-05), §3:
 *               32-element blocks, scale maps the block max to the FP4 max.
 *   [MR-GPTQ]   "FP4 quantization analysis: MXFP4 vs NVFP4" (jsqmd.com),
 *               §3.2.3: block-diagonal Hadamard H_k, k in {16,32,64,128};
 *               §3.2.1: block scales chosen to minimise the squared error
 *               sum ||Y^_i - X_i||^2; §3.3: "MSE" and "Abs-Max" methods.
 *   [gpt-oss]   "gpt-oss MXFP4" article (juejin.cn), MXFP4 section: the
 *               worked example 0.0625, 0.375, 0.078125, 0.25.
 *
 * Readings where the pages are silent (each one also listed in the design
 * notes): E2M1 ties either to the even code (default) or away from zero;
 * MXFP4 scale exponent = the smallest power of two that keeps the block
 * max <= 6 (default) or the OCP floor rule; E8M0 bias 127; NVFP4 global
 * scale s_g = amax/(6*448); one reciprocal per NVFP4 block, then a multiply;
 * the rotation is the normalised Sylvester FWHT along K, stages h ascending;
 * the MSE method searches a fixed window of scales around the absmax one
 * and compares fp32 block errors summed in a fixed pairwise order.
 */
#include "fp4_oracle.h"

#include <float.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* Element format E2M1 ([Guide] §3.1): 1 sign, 2 exponent, 1 mantissa bit.   */
/* Code c (0..7) of the magnitude: exponent bits = c>>1, mantissa bit = c&1, */
/* bias 1, exponent 0 is subnormal (0 or 0.5).  Largest value 2^2*1.5 = 6.   */
/* ------------------------------------------------------------------------ */
static double e2m1_magnitude(int c)
{
    int ebits = (c >> 1) & 3, mbit = c & 1;
    if (ebits == 0) return 0.5 * mbit;                      /* subnormal */
    return ldexp(1.0 + 0.5 * mbit, ebits - 1);
}

double fp4o_e2m1_decode(int code)
{
    double m = e2m1_magnitude(code & 7);
    return (code & 8) ? -m : m;
}

/* Nearest-value encode of v ([TransFP4] §3.1 "nearest rounding").  |v| >= 6
 * (including +inf) saturates to the largest code.  At an exact midpoint the
 * tie goes to the even code (mantissa bit 0) or to the larger magnitude.
 * The sign is copied from v, so -0 and negatives that round to 0 give 0x8. */
int fp4o_e2m1_encode(float v, int tie)
{
    int sign = signbit(v) ? 8 : 0;
    double a = fabs((double)v);
    if (!(a < 6.0)) return sign | 7;                        /* sat / inf */
    int lo = 0;
    while (lo < 7 && e2m1_magnitude(lo + 1) <= a) lo++;     /* g[lo] <= a */
    int hi = lo + 1;
    double dlo = a - e2m1_magnitude(lo), dhi = e2m1_magnitude(hi) - a;
    int c;
    if (dlo < dhi) c = lo;
    else if (dhi < dlo) c = hi;
    else c = (tie == FP4O_TIE_AWAY) ? hi : ((lo & 1) ? hi : lo);
    return sign | c;
}

/* ------------------------------------------------------------------------ */
/* Scale format E4M3, unsigned use ([Guide] §1.1-1.2): exponent 4 bits,      */
/* bias 7, mantissa 3 bits, subnormals at exponent 0, largest finite 448     */
/* (0x7E); 0x7F is NaN and no infinity exists.                               */
/* ------------------------------------------------------------------------ */
double fp4o_e4m3_decode(int byte)
{
    int b = byte & 0x7F;
    if (b == 0x7F) return NAN;
    int e = b >> 3, m = b & 7;
    if (e == 0) return ldexp((double)m, -9);                /* m/8 * 2^-6 */
    return ldexp(1.0 + m / 8.0, e - 7);
}

/* Round-to-nearest-even onto the 127 finite non-negative codes, saturating
 * at 448.  t must be >= 0 (block scales are non-negative). */
int fp4o_e4m3_encode(float t)
{
    double a = (double)t;
    if (!(a < 448.0)) return 0x7E;                          /* satfinite */
    int best = 0;
    double bestd = fabs(a - fp4o_e4m3_decode(0));
    for (int c = 1; c <= 0x7E; c++) {
        double d = fabs(a - fp4o_e4m3_decode(c));
        if (d < bestd || (d == bestd && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            bestd = d;
        }
    }
    return best;
}

/* E8M0: power-of-two scale 2^(byte-127) ([TransFP4] §1.1, [Guide] §3.3);
 * 0xFF is NaN. */
double fp4o_e8m0_decode(int byte)
{
    if ((byte & 0xFF) == 0xFF) return NAN;
    return ldexp(1.0, (byte & 0xFF) - 127);
}

/* MXFP4 shared exponent of a block with largest magnitude amax.
 * CEIL (default): the smallest e with amax <= 6 * 2^e, i.e. the block max
 *   is mapped onto the E2M1 range without clipping ([Explainer] §3).
 * FLOOR (option): e = floor(log2 amax) - 2 (the OCP MX rule; block values
 *   in (6, 8) * 2^e saturate to 6).
 * amax == 0 gives -127 (byte 0x00).  The result is clamped to [-127, 127]. */
int fp4o_mx_scale_exponent(float amax, int rule)
{
    if (amax == 0.0f) return -127;
    int p;
    double f = frexp((double)amax, &p);                     /* amax = f*2^p */
    (void)f;
    int e;
    if (rule == FP4O_MX_FLOOR) {
        e = (p - 1) - 2;                                    /* floor(log2) = p-1 */
    } else {
        /* amax > 2^(p-1) >= 6*2^(p-4), so no e below p-4 can satisfy the bound:
         * search upward from there. */
        e = p - 4;
        while (!((double)amax <= ldexp(6.0, e))) e++;
    }
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

/* ------------------------------------------------------------------------ */
/* Block-diagonal Hadamard rotation H_k ([MR-GPTQ] §3.2.3; [TransFP4] §2.3)  */
/* ------------------------------------------------------------------------ */
float fp4o_hadamard_ck(int k)
{
    return (float)(1.0 / sqrt((double)k));
}

/* Normalised Sylvester Walsh-Hadamard transform of one chunk of k values,
 * in place, in fp32: stages h = 1, 2, ..., k/2 replace each pair
 * (y[j], y[j+h]) (bit h of j clear) by (y[j] + y[j+h], y[j] - y[j+h]); then
 * every value is multiplied by c_k = RN(1/sqrt(k)).  The matrix is
 * symmetric and orthogonal, so applying it twice returns the input up to
 * rounding. */
void fp4o_fwht(float *y, int k)
{
    for (int h = 1; h < k; h *= 2) {
        for (int j = 0; j < k; j++) {
            if (j & h) continue;
            float a = y[j], b = y[j + h];
            y[j] = a + b;
            y[j + h] = a - b;
        }
    }
    float ck = fp4o_hadamard_ck(k);
    for (int j = 0; j < k; j++) y[j] = y[j] * ck;
}

/* ------------------------------------------------------------------------ */
/* Quantize ([TransFP4] Eq.(1): x^_i = s_g s_b Q_f(x_i / (s_g s_b)))         */
/* ------------------------------------------------------------------------ */
static float bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static int valid_shape(int fmt, int block, int hk, int64_t rows, int64_t cols)
{
    if (rows < 0 || cols < 0) return 0;
    /* MXFP4 also on 16-element blocks: the microscaling form of [TransFP4]
     * §1.1 leaves the block size G open, and E8M0 scales on 16-element blocks
     * separate the block-size effect from the scale-precision effect that
     * tell MXFP4 and NVFP4 apart ([Guide] §3.3). */
    if (fmt == FP4O_MXFP4 && block != 32 && block != 16) return 0;
    if (fmt == FP4O_NVFP4 && block != 16) return 0;
    if (fmt != FP4O_MXFP4 && fmt != FP4O_NVFP4) return 0;
    if (!(hk == 0 || hk == 16 || hk == 32 || hk == 64 || hk == 128)) return 0;
    if (cols % block) return 0;
    if (hk && cols % hk) return 0;
    return 1;
}

/* Row r of x as fp32, rotated when hk > 0. */
/* One row of the input, as fp32: either bf16 elements (xb) or fp32 elements
 * (xf, e.g. a product that is quantized again for the next layer); then the
 * rotation, if any. */
static void load_row(const uint16_t *xb, const float *xf, int64_t ld, int64_t r,
                     int64_t cols, int hk, float *y)
{
    for (int64_t c = 0; c < cols; c++)
        y[c] = xb ? bf16_to_f32(xb[r * ld + c]) : xf[r * ld + c];
    if (hk)
        for (int64_t c = 0; c < cols; c += hk) fp4o_fwht(y + c, hk);
}

/* NVFP4 tensor scale ([Guide] §4.1: the FP32 tensor-level scale brings the
 * tensor into the E4M3 block-scale range): s_g = amax / (6 * 448), so the
 * largest block scale lands at the E4M3 maximum; an all-zero tensor (or a
 * non-finite amax) gets s_g = 1. */
static float nv_global_scale(float amax_t)
{
    if (amax_t > 0.0f && amax_t <= FLT_MAX) return amax_t / 2688.0f;
    return 1.0f;
}

/* bf16 bit pattern of an fp32 value, rounded to nearest, ties to even (the
 * precision of the residual lane). */
static uint16_t f32_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x7FFFFFu)) return (uint16_t)((u >> 16) | 0x40);  /* NaN */
    uint32_t lsb = (u >> 16) & 1u;
    return (uint16_t)((u + 0x7FFFu + lsb) >> 16);
}

/* Sparse residual lane ([TransFP4] §2.3 Eq.(3), r = 1 per 32 values): in
 * every 32-value unit of the rotated row y, the value of largest magnitude
 * (the first of equal ones) leaves the FP4 stream: it is kept as a bf16 value
 * with its 5-bit position (word = bf16 bits | index << 16) and zeroed in y,
 * which is then quantized as usual. */
static void extract_residuals(float *y, int64_t cols, uint32_t *res_row)
{
    for (int64_t u = 0; u < cols / 32; u++) {
        float *v = y + u * 32;
        int best = 0;
        for (int i = 1; i < 32; i++)
            if (fabsf(v[i]) > fabsf(v[best])) best = i;
        if (res_row) res_row[u] = (uint32_t)f32_to_bf16_rne(v[best]) | ((uint32_t)best << 16);
        v[best] = 0.0f;
    }
}

/* The absmax scale byte of one block ([TransFP4] §3.1): MX the E8M0 byte of
 * fp4o_mx_scale_exponent(amax, rule); NV the E4M3 code of t = amax / (6 s_g). */
static int absmax_scale_byte(const float *blk, int block, int fmt, int mx_rule, float sg)
{
    float amax_b = 0.0f;
    for (int i = 0; i < block; i++)
        if (fabsf(blk[i]) > amax_b) amax_b = fabsf(blk[i]);
    if (fmt == FP4O_MXFP4) return fp4o_mx_scale_exponent(amax_b, mx_rule) + 127;
    float six_sg = 6.0f * sg;
    return fp4o_e4m3_encode(amax_b / six_sg);
}

/* Elements of one block under a given scale byte ([TransFP4] Eq.(1),
 * q_i = Q_f(x_i / d)).  MX: d = 2^e, and x / 2^e is the exact product
 * x * 2^-e.  NV: d = s_g * s_b, the values are multiplied by r = 1/d
 * (clamped to the largest float); d = 0 gives signed zeros. */
static void encode_block(const float *blk, int block, int fmt, int sbyte, float sg, int tie,
                         int *codes)
{
    if (fmt == FP4O_MXFP4) {
        float inv = ldexpf(1.0f, -(sbyte - 127));
        for (int i = 0; i < block; i++) codes[i] = fp4o_e2m1_encode(blk[i] * inv, tie);
        return;
    }
    float d = sg * (float)fp4o_e4m3_decode(sbyte);
    if (d == 0.0f) {
        for (int i = 0; i < block; i++) codes[i] = signbit(blk[i]) ? 8 : 0;
        return;
    }
    float rcp = 1.0f / d;
    if (rcp > FLT_MAX) rcp = FLT_MAX;
    for (int i = 0; i < block; i++) codes[i] = fp4o_e2m1_encode(blk[i] * rcp, tie);
}

/* Squared reconstruction error of one encoded block ([MR-GPTQ] §3.2.1,
 * sum_i (Y^_i - X_i)^2 with Y^_i = d * q_i), one fp32 operation per step:
 * y_i = RN(q_i * d), e_i = RN(x_i - y_i), e_i^2 rounded; then a fixed
 * pairwise sum: adjacent pairs first, then the first half of the partial
 * sums plus the second half, until one value remains. */
static float block_sse(const float *blk, int block, int fmt, int sbyte, float sg, const int *codes)
{
    float d = (fmt == FP4O_MXFP4) ? ldexpf(1.0f, sbyte - 127) : sg * (float)fp4o_e4m3_decode(sbyte);
    float t[32];
    for (int i = 0; i < block; i++) {
        float y = (float)fp4o_e2m1_decode(codes[i]) * d;
        float e = blk[i] - y;
        t[i] = e * e;
    }
    for (int i = 0; i < block / 2; i++) t[i] = t[2 * i] + t[2 * i + 1];
    for (int w = block / 4; w >= 1; w /= 2)
        for (int i = 0; i < w; i++) t[i] = t[i] + t[i + w];
    return t[0];
}

/* The "MSE" method ([MR-GPTQ] §3.2.1, §3.3): of a short list of candidate
 * scales around the absmax one, the block takes the one whose encoding has
 * the smallest block_sse; of equal ones the first.  Candidates, in order:
 *   MX: e_c, then e_c - 1 (above -127 only), e_c the CEIL exponent; the
 *       FLOOR rule's exponent is one of the two.  Larger exponents only
 *       coarsen the grid; smaller ones clip the block max to half or less.
 *   NV: t0, then t0 - 2, t0 - 1, t0 + 1, ..., t0 + 6, t0 the absmax E4M3
 *       code; only codes 1 .. 0x7E (0x7F is NaN, 0 zeroes the block).  The
 *       window maps the block max to between about 3.6 and 7.3 on the E2M1
 *       grid: below 6 the top of the grid (spacing 2 between 4 and 6) may
 *       serve the largest values of a block better.
 * Writes the chosen block's codes and returns its scale byte. */
static int mse_scale_byte(const float *blk, int block, int fmt, float sg, int tie, int *codes)
{
    int cand[9], nc = 0;
    int s0 = absmax_scale_byte(blk, block, fmt, FP4O_MX_CEIL, sg);
    cand[nc++] = s0;
    if (fmt == FP4O_MXFP4) {
        if (s0 > 0) cand[nc++] = s0 - 1;
    } else {
        for (int j = -2; j <= 6; j++)
            if (j != 0 && s0 + j >= 1 && s0 + j <= 0x7E) cand[nc++] = s0 + j;
    }
    int best = -1;
    float best_sse = 0.0f;
    int trial[32];
    for (int c = 0; c < nc; c++) {
        encode_block(blk, block, fmt, cand[c], sg, tie, trial);
        float e = block_sse(blk, block, fmt, cand[c], sg, trial);
        if (best < 0 || e < best_sse) {
            best = cand[c];
            best_sse = e;
            memcpy(codes, trial, sizeof(int) * (size_t)block);
        }
    }
    return best;
}

static int quantize_rows(const uint16_t *xb, const float *xf, int64_t rows, int64_t cols,
                         int64_t ld, int fmt, int block, int hadamard_k, int tie,
                         int mx_rule, int search, int gscale_given, float *gscale, uint8_t *q,
                         uint8_t *s_logical, uint32_t *res)
{
    if (!valid_shape(fmt, block, hadamard_k, rows, cols) || ld < cols) return -1;
    if (search != FP4O_SCALE_ABSMAX && search != FP4O_SCALE_MSE) return -1;
    const int64_t nkb = cols / block;

    float sg = 1.0f;
    if (fmt == FP4O_NVFP4) {
        if (gscale_given) {
            sg = *gscale;
        } else {
            float amax_t = 0.0f;
#pragma omp parallel
            {
                float *y = (float *)malloc(sizeof(float) * (size_t)(cols ? cols : 1));
                float local = 0.0f;
#pragma omp for schedule(static)
                for (int64_t r = 0; r < rows; r++) {
                    load_row(xb, xf, ld, r, cols, hadamard_k, y);
                    if (res) extract_residuals(y, cols, NULL);  /* s_g of the FP4 stream */
                    for (int64_t c = 0; c < cols; c++) {
                        float a = fabsf(y[c]);
                        if (a > local) local = a;
                    }
                }
#pragma omp critical
                if (local > amax_t) amax_t = local;
                free(y);
            }
            sg = nv_global_scale(amax_t);
            *gscale = sg;
        }
    }

#pragma omp parallel
    {
        float *y = (float *)malloc(sizeof(float) * (size_t)(cols ? cols : 1));
#pragma omp for schedule(static)
        for (int64_t r = 0; r < rows; r++) {
            load_row(xb, xf, ld, r, cols, hadamard_k, y);
            if (res) extract_residuals(y, cols, res + r * (cols / 32));
            uint8_t *qrow = q + r * (cols / 2);
            memset(qrow, 0, (size_t)(cols / 2));
            for (int64_t kb = 0; kb < nkb; kb++) {
                const float *blk = y + kb * block;
                int codes[32];
                int sbyte;
                if (search == FP4O_SCALE_MSE) {
                    sbyte = mse_scale_byte(blk, block, fmt, sg, tie, codes);
                } else {
                    sbyte = absmax_scale_byte(blk, block, fmt, mx_rule, sg);
                    encode_block(blk, block, fmt, sbyte, sg, tie, codes);
                }
                s_logical[r * nkb + kb] = (uint8_t)sbyte;
                for (int i = 0; i < block; i++) {
                    int64_t c = kb * block + i;
                    qrow[c / 2] |= (uint8_t)((codes[i] & 0xF) << ((c & 1) ? 4 : 0));
                }
            }
        }
        free(y);
    }
    return 0;
}

int fp4o_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                  int fmt, int block, int hadamard_k, int tie, int mx_rule, int search,
                  int gscale_given, float *gscale,
                  uint8_t *q, uint8_t *s_logical)
{
    return quantize_rows(x, NULL, rows, cols, ld, fmt, block, hadamard_k, tie, mx_rule,
                         search, gscale_given, gscale, q, s_logical, NULL);
}

/* Alternating refinement of the NVFP4 tensor scale ([MR-GPTQ] §3.2.1: the
 * group scales and the tensor scale are optimised in turn for the smallest
 * sum ||Y^_i - X_i||^2).  Starting from the absmax s_g, each round
 *   (group step)  quantizes the rotated tensor with the MSE block-scale
 *                 search under the current s_g;
 *   (evaluation)  E = sum (x_i - y_i)^2 over the rotated values x_i and
 *                 their reconstructions y_i = RN(RN(s_g dec(s_b)) dec(q_i));
 *   (global step) s_g <- RN_fp32(sum x_i u_i / sum u_i^2), u_i = dec(s_b)
 *                 dec(q_i): the least-squares tensor scale for the codes
 *                 just chosen (kept when the sum of u_i^2 is 0 or the
 *                 quotient is not a positive finite float).
 * After `rounds` evaluations the s_g with the smallest E (the first of equal
 * ones) is returned, with E.  Sums are fp64 in a fixed order: over the 32
 * values of a unit in index order, over a row's units in order, then over
 * the rows in order; products x_i u_i and u_i^2 are exact in fp64. */
int fp4o_nv_refine_gscale(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                          int hadamard_k, int tie, int rounds, float *gscale, double *err)
{
    if (!valid_shape(FP4O_NVFP4, 16, hadamard_k, rows, cols) || ld < cols || rounds < 1) return -1;
    const int64_t nkb = cols / 16, units = cols / 32;
    uint8_t *q = (uint8_t *)calloc((size_t)(rows * (cols / 2) + 1), 1);
    uint8_t *s = (uint8_t *)calloc((size_t)(rows * nkb + 1), 1);
    float *y = (float *)malloc(sizeof(float) * (size_t)(cols ? cols : 1));
    double *row_xu = (double *)malloc(sizeof(double) * (size_t)(rows ? rows : 1));
    double *row_uu = (double *)malloc(sizeof(double) * (size_t)(rows ? rows : 1));
    double *row_ee = (double *)malloc(sizeof(double) * (size_t)(rows ? rows : 1));
    float sg = 0.0f;
    /* the absmax s_g, as fp4o_quantize computes it */
    quantize_rows(x, NULL, rows, cols, ld, FP4O_NVFP4, 16, hadamard_k, tie, FP4O_MX_CEIL,
                  FP4O_SCALE_ABSMAX, 0, &sg, q, s, NULL);
    float best_sg = sg;
    double best_e = 0.0;
    for (int t = 0; t < rounds; t++) {
        float cur = sg;
        quantize_rows(x, NULL, rows, cols, ld, FP4O_NVFP4, 16, hadamard_k, tie, FP4O_MX_CEIL,
                      FP4O_SCALE_MSE, 1, &cur, q, s, NULL);
        for (int64_t r = 0; r < rows; r++) {
            load_row(x, NULL, ld, r, cols, hadamard_k, y);
            double rxu = 0.0, ruu = 0.0, ree = 0.0;
            for (int64_t u = 0; u < units; u++) {
                double uxu = 0.0, uuu = 0.0, uee = 0.0;
                for (int i = 0; i < 32; i++) {
                    int64_t c = u * 32 + i;
                    int code = (q[r * (cols / 2) + c / 2] >> ((c & 1) ? 4 : 0)) & 0xF;
                    int sb = s[r * nkb + c / 16];
                    double ui = fp4o_e4m3_decode(sb) * fp4o_e2m1_decode(code);
                    float d = sg * (float)fp4o_e4m3_decode(sb);
                    float yi = d * (float)fp4o_e2m1_decode(code);
                    double e = (double)y[c] - (double)yi;
                    uxu = uxu + (double)y[c] * ui;
                    uuu = uuu + ui * ui;
                    uee = uee + e * e;
                }
                rxu = rxu + uxu;
                ruu = ruu + uuu;
                ree = ree + uee;
            }
            row_xu[r] = rxu;
            row_uu[r] = ruu;
            row_ee[r] = ree;
        }
        double sxu = 0.0, suu = 0.0, see = 0.0;
        for (int64_t r = 0; r < rows; r++) {
            sxu = sxu + row_xu[r];
            suu = suu + row_uu[r];
            see = see + row_ee[r];
        }
        if (t == 0 || see < best_e) {
            best_e = see;
            best_sg = sg;
        }
        if (suu > 0.0) {
            float nxt = (float)(sxu / suu);
            if (nxt > 0.0f && nxt <= FLT_MAX) sg = nxt;
        }
    }
    *gscale = best_sg;
    if (err) *err = best_e;
    free(q);
    free(s);
    free(y);
    free(row_xu);
    free(row_uu);
    free(row_ee);
    return 0;
}

int fp4o_quantize_residual(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                           int fmt, int block, int hadamard_k, int tie, int mx_rule,
                           int gscale_given, float *gscale, uint8_t *q, uint8_t *s_logical,
                           uint32_t *res)
{
    if (!res) return -1;
    return quantize_rows(x, NULL, rows, cols, ld, fmt, block, hadamard_k, tie, mx_rule,
                         FP4O_SCALE_ABSMAX, gscale_given, gscale, q, s_logical, res);
}

int fp4o_quantize_f32(const float *x, int64_t rows, int64_t cols, int64_t ld,
                      int fmt, int block, int hadamard_k, int tie, int mx_rule, int search,
                      int gscale_given, float *gscale,
                      uint8_t *q, uint8_t *s_logical)
{
    return quantize_rows(NULL, x, rows, cols, ld, fmt, block, hadamard_k, tie, mx_rule,
                         search, gscale_given, gscale, q, s_logical, NULL);
}

/* ------------------------------------------------------------------------ */
/* Dequantize ([TransFP4] Eq.(1); [Guide] §4.1 x^ = s_tensor * s_block * q)  */
/* ------------------------------------------------------------------------ */
static int dequantize_rows(const uint8_t *q, const uint8_t *s_logical, float gscale,
                           const uint32_t *res, int64_t rows, int64_t cols, int fmt, int block,
                           int hadamard_k, float *out)
{
    if (!valid_shape(fmt, block, hadamard_k, rows, cols)) return -1;
    const int64_t nkb = cols / block;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        float *o = out + r * cols;
        for (int64_t c = 0; c < cols; c++) {
            int code = (q[r * (cols / 2) + c / 2] >> ((c & 1) ? 4 : 0)) & 0xF;
            float qv = (float)fp4o_e2m1_decode(code);
            uint8_t sb = s_logical[r * nkb + c / block];
            if (fmt == FP4O_MXFP4) {
                o[c] = qv * (float)fp4o_e8m0_decode(sb);
            } else {
                float d = gscale * (float)fp4o_e4m3_decode(sb);
                o[c] = d * qv;
            }
        }
        if (res)  /* [TransFP4] Eq.(3): the FP4 stream plus the residual lane */
            for (int64_t u = 0; u < cols / 32; u++) {
                uint32_t w = res[r * (cols / 32) + u];
                o[u * 32 + ((w >> 16) & 31)] += bf16_to_f32((uint16_t)(w & 0xFFFFu));
            }
        if (hadamard_k)
            for (int64_t c = 0; c < cols; c += hadamard_k) fp4o_fwht(o + c, hadamard_k);
    }
    return 0;
}

int fp4o_dequantize(const uint8_t *q, const uint8_t *s_logical, float gscale,
                    int64_t rows, int64_t cols, int fmt, int block,
                    int hadamard_k, float *out)
{
    return dequantize_rows(q, s_logical, gscale, NULL, rows, cols, fmt, block, hadamard_k, out);
}

int fp4o_dequantize_residual(const uint8_t *q, const uint8_t *s_logical, float gscale,
                             const uint32_t *res, int64_t rows, int64_t cols, int fmt, int block,
                             int hadamard_k, float *out)
{
    if (!res) return -1;
    return dequantize_rows(q, s_logical, gscale, res, rows, cols, fmt, block, hadamard_k, out);
}

/* ------------------------------------------------------------------------ */
/* MXFP4 -> NVFP4 scale repacking ([TransFP4] §2.5 and §3.4: a logical       */
/* artifact is bound late to the backend's native format; "NVFP4 activations */
/* with MXFP4 weights" needs the weights in the NVFP4 scale form).  The      */
/* E2M1 elements are kept; each 32-block power-of-two scale 2^e becomes two  */
/* 16-block E4M3 scales 2^(e - E) under the tensor scale s_g = 2^E, so that  */
/* s_g * s_b = 2^e and every element dequantizes to the same value          */
/* ([Guide] §4.1).  E = max(e_max - 8, -126): the largest block scale lands  */
/* on 2^8, the largest power of two E4M3 holds, and s_g stays a normal       */
/* float.  Blocks more than 17 binades below the largest (2^(e-E) below the  */
/* smallest E4M3 subnormal 2^-9) take the E4M3 rounding of 2^(e-E): 0.       */
/* E8M0 NaN (0xFF) maps to E4M3 NaN (0x7F).                                   */
/* ------------------------------------------------------------------------ */
int fp4o_mx_scales_to_nv(const uint8_t *s_mx, int64_t rows, int64_t nkb, uint8_t *s_nv,
                         float *gscale)
{
    if (rows < 0 || nkb < 0) return -1;
    int e_max = -1000;
    for (int64_t i = 0; i < rows * nkb; i++)
        if (s_mx[i] != 0xFF && (int)s_mx[i] - 127 > e_max) e_max = (int)s_mx[i] - 127;
    int E = e_max - 8;
    if (E < -126) E = -126;
    *gscale = ldexpf(1.0f, E);
    for (int64_t r = 0; r < rows; r++)
        for (int64_t kb = 0; kb < nkb; kb++) {
            uint8_t b = s_mx[r * nkb + kb];
            uint8_t nv = (b == 0xFF) ? 0x7F : (uint8_t)fp4o_e4m3_encode(ldexpf(1.0f, (int)b - 127 - E));
            s_nv[r * 2 * nkb + 2 * kb] = nv;
            s_nv[r * 2 * nkb + 2 * kb + 1] = nv;
        }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* INT4 group quantization, the INT4 baseline of [TransFP4] Table 5 (§3.1:   */
/* every method uses per-block absmax scales and nearest rounding).  A group */
/* of G consecutive values takes the fp32 scale s = amax / 7 and the integer */
/* codes q_i = x_i / s rounded to nearest (ties to even), clamped to         */
/* [-7, 7]; an all-zero group has s = 0 and codes 0.  x^_i = q_i * s.         */
/* ------------------------------------------------------------------------ */
static float int4_group(const float *x, int G, int8_t *q)
{
    float amax = 0.0f;
    for (int i = 0; i < G; i++)
        if (fabsf(x[i]) > amax) amax = fabsf(x[i]);
    float s = amax / 7.0f;
    for (int i = 0; i < G; i++) {
        float v = (s == 0.0f) ? 0.0f : nearbyintf(x[i] / s);
        if (v > 7.0f) v = 7.0f;
        if (v < -7.0f) v = -7.0f;
        q[i] = (int8_t)v;
    }
    return s;
}

int fp4o_int4_quantize_f32(const float *x, int64_t rows, int64_t cols, int group, int8_t *q,
                           float *scales)
{
    if (rows < 0 || cols < 0 || group < 2 || cols % group) return -1;
    const int64_t ng = cols / group;
    for (int64_t r = 0; r < rows; r++)
        for (int64_t g = 0; g < ng; g++)
            scales[r * ng + g] = int4_group(x + r * cols + g * group, group, q + r * cols + g * group);
    return 0;
}

int fp4o_int4_dequantize(const int8_t *q, const float *scales, int64_t rows, int64_t cols, int group,
                         float *out)
{
    if (rows < 0 || cols < 0 || group < 2 || cols % group) return -1;
    const int64_t ng = cols / group;
    for (int64_t r = 0; r < rows; r++)
        for (int64_t c = 0; c < cols; c++) out[r * cols + c] = (float)q[r * cols + c] * scales[r * ng + c / group];
    return 0;
}

/* ------------------------------------------------------------------------ */
/* The TransFP4 method as the page's numerical experiment runs it ([TransFP4] */
/* §2.3 Eq.(2)-(3), §3.1): rotate every k-chunk (H_k; the page uses k = 32),  */
/* take the largest-magnitude value of each 32-value unit out as the bf16     */
/* residual lane, and quantize each unit with the better of two candidates   */
/* by its block error: NVFP4 (two 16-blocks, absmax E4M3 scales under the    */
/* tensor scale s_g of the remaining values) or INT4 (one 32-value group).   */
/* Per unit: e_c = sum (y_i - y^_i)^2 in fp64 over the unit's rotated values  */
/* y (the residual position zeroed); INT4 only if its e is strictly smaller  */
/* (NVFP4 always with allow_int4 = 0).  x^ = the chosen reconstruction plus  */
/* the residual value at its position, rotated back.  choice[u] = 0 NVFP4,    */
/* 1 INT4.  The per-unit 2-bit format tag of the page's IR is this choice.    */
/* ------------------------------------------------------------------------ */
int fp4o_transfp4_f32(const float *x, int64_t rows, int64_t cols, int hadamard_k, int tie,
                      int allow_int4, float *out, uint8_t *choice)
{
    if (!valid_shape(FP4O_NVFP4, 16, hadamard_k, rows, cols) || cols % 32) return -1;
    float *y = (float *)malloc(sizeof(float) * (size_t)(cols ? cols : 1));
    uint32_t *res = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)(cols / 32 + 1));
    if (!y || !res) {
        free(y);
        free(res);
        return -1;
    }
    /* s_g of the FP4 stream: the maximum over the values left after the
     * residual lane */
    float amax_t = 0.0f;
    for (int64_t r = 0; r < rows; r++) {
        load_row(NULL, x, cols, r, cols, hadamard_k, y);
        extract_residuals(y, cols, NULL);
        for (int64_t c = 0; c < cols; c++)
            if (fabsf(y[c]) > amax_t) amax_t = fabsf(y[c]);
    }
    const float sg = nv_global_scale(amax_t);
    for (int64_t r = 0; r < rows; r++) {
        load_row(NULL, x, cols, r, cols, hadamard_k, y);
        extract_residuals(y, cols, res);
        float *o = out + r * cols;
        for (int64_t u = 0; u < cols / 32; u++) {
            const float *v = y + u * 32;
            float nv[32], i4[32];
            for (int b = 0; b < 2; b++) {
                int codes[16];
                const int sb = absmax_scale_byte(v + 16 * b, 16, FP4O_NVFP4, FP4O_MX_CEIL, sg);
                encode_block(v + 16 * b, 16, FP4O_NVFP4, sb, sg, tie, codes);
                const float d = sg * (float)fp4o_e4m3_decode(sb);
                for (int i = 0; i < 16; i++) nv[16 * b + i] = d * (float)fp4o_e2m1_decode(codes[i]);
            }
            int8_t q4[32];
            const float s4 = int4_group(v, 32, q4);
            for (int i = 0; i < 32; i++) i4[i] = (float)q4[i] * s4;
            double e_nv = 0.0, e_i4 = 0.0;
            for (int i = 0; i < 32; i++) {
                e_nv += ((double)v[i] - nv[i]) * ((double)v[i] - nv[i]);
                e_i4 += ((double)v[i] - i4[i]) * ((double)v[i] - i4[i]);
            }
            const int pick = allow_int4 && e_i4 < e_nv;
            choice[r * (cols / 32) + u] = (uint8_t)pick;
            for (int i = 0; i < 32; i++) o[u * 32 + i] = pick ? i4[i] : nv[i];
            o[u * 32 + ((res[u] >> 16) & 31)] += bf16_to_f32((uint16_t)(res[u] & 0xFFFFu));
        }
        if (hadamard_k)
            for (int64_t c = 0; c < cols; c += hadamard_k) fp4o_fwht(o + c, hadamard_k);
    }
    free(y);
    free(res);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Scale tile layout consumed by the block-scaled tensor-core MMA: 512-byte   */
/* atoms of 128 rows x 4 scale columns; atoms ordered row-block major, then  */
/* scale-column block.  Inside an atom, row r and column j sit at byte       */
/* (r % 32) * 16 + (r / 32) * 4 + j.  Rows pad to 128, columns to 4; padding */
/* bytes are 0.  (A hardware convention; the pages do not fix it.)           */
/* ------------------------------------------------------------------------ */
static int64_t atom_offset(int64_t r, int64_t kb, int64_t nkb4)
{
    return ((r / 128) * nkb4 + kb / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (kb % 4);
}

void fp4o_scales_to_atoms(const uint8_t *s_logical, int64_t rows, int64_t nkb,
                          uint8_t *s_atoms)
{
    int64_t rows_p = (rows + 127) / 128 * 128, nkb4 = (nkb + 3) / 4;
    memset(s_atoms, 0, (size_t)(rows_p * nkb4 * 4));
    for (int64_t r = 0; r < rows; r++)
        for (int64_t kb = 0; kb < nkb; kb++)
            s_atoms[atom_offset(r, kb, nkb4)] = s_logical[r * nkb + kb];
}

void fp4o_scales_from_atoms(const uint8_t *s_atoms, int64_t rows, int64_t nkb,
                            uint8_t *s_logical)
{
    int64_t nkb4 = (nkb + 3) / 4;
    for (int64_t r = 0; r < rows; r++)
        for (int64_t kb = 0; kb < nkb; kb++)
            s_logical[r * nkb + kb] = s_atoms[atom_offset(r, kb, nkb4)];
}

/* ------------------------------------------------------------------------ */
/* W4A4 linear reference: C = A_hat * W_hat^T in fp64 over the dequantized   */
/* operands ([Guide] §5: the product of quantized activations and weights).  */
/* ------------------------------------------------------------------------ */
void fp4o_gemm_ref(const float *a, const float *w, int64_t M, int64_t N,
                   int64_t K, double *c, double *bound)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; m++) {
        for (int64_t n = 0; n < N; n++) {
            double acc = 0.0, acc_abs = 0.0;
            for (int64_t k = 0; k < K; k++) {
                double p = (double)a[m * K + k] * (double)w[n * K + k];
                acc += p;
                acc_abs += fabs(p);
            }
            c[m * N + n] = acc;
            if (bound) bound[m * N + n] = acc_abs;
        }
    }
}

int fp4o_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
