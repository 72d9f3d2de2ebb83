/*
 * fp4_oracle.h — plain, slow CPU oracle for microscaling FP4 quantization
 * and the block-scaled W4A4 product.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link
 * or call this library; only the test-suite, the smoke check and the CPU
 * baseline leg of the benchmark load it.  It shares no code, header, table
 * or constant with the CUDA library under fp4_microscaling_quantization_b200/.
 *
 * Conventions (all functions):
 *   - Every fp32 operation is a single IEEE-754 binary32 operation rounded to
 *     nearest-even (the build uses -ffp-contract=off and no fast-math, so no
 *     operation is fused or reassociated).  Subnormals are kept.
 *   - Elements are bf16 bit patterns (uint16_t), rows x cols, row stride ld
 *     (in elements).  The quantization / contraction axis is cols (K).
 *   - fmt/block: FP4O_MXFP4 with block 32 or 16 (E8M0 scales), FP4O_NVFP4
 *     with block 16 (E4M3 scales under an fp32 tensor scale).
 *   - Scales are returned in LOGICAL layout: s[row * (cols/block) + kb].
 *     The hardware tile layout is produced by fp4o_scales_to_atoms().
 *   - Packed elements: byte (row, j) holds element 2j in bits [3:0] and
 *     element 2j+1 in bits [7:4]; row stride cols/2 bytes.
 */
#ifndef FP4_ORACLE_H
#define FP4_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { FP4O_MXFP4 = 0, FP4O_NVFP4 = 1 };
enum { FP4O_TIE_EVEN = 0, FP4O_TIE_AWAY = 1 };
enum { FP4O_MX_CEIL = 0, FP4O_MX_FLOOR = 1 };
enum { FP4O_SCALE_ABSMAX = 0, FP4O_SCALE_MSE = 1 };

/* ---- element and scale codecs ------------------------------------------- */
int    fp4o_e2m1_encode(float v, int tie);      /* 4-bit code, sign in bit 3 */
double fp4o_e2m1_decode(int code);
int    fp4o_e4m3_encode(float t);               /* t >= 0, RNE, satfinite    */
double fp4o_e4m3_decode(int byte);
double fp4o_e8m0_decode(int byte);              /* 2^(byte-127); NaN at 0xFF */
int    fp4o_mx_scale_exponent(float amax, int rule);  /* e in [-127, 127]    */

/* ---- rotation ----------------------------------------------------------- */
float  fp4o_hadamard_ck(int k);                 /* RN_fp32(1/sqrt(k))        */
void   fp4o_fwht(float *y, int k);              /* in place, incl. c_k       */

/* ---- quantize / dequantize --------------------------------------------- */
/* gscale: NVFP4 only.  If gscale_given, *gscale is read as s_g; otherwise
 * s_g is computed from the tensor and written to *gscale.  search: block
 * scale by absmax (mx_rule applies) or by the MSE search over the absmax
 * scale's neighbours (mx_rule ignored).  Returns 0 on success, -1 on an
 * invalid argument. */
int fp4o_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                  int fmt, int block, int hadamard_k, int tie, int mx_rule, int search,
                  int gscale_given, float *gscale,
                  uint8_t *q, uint8_t *s_logical);

/* The same with fp32 elements (row stride ld floats): a product quantized
 * again, e.g. for the next layer. */
int fp4o_quantize_f32(const float *x, int64_t rows, int64_t cols, int64_t ld,
                      int fmt, int block, int hadamard_k, int tie, int mx_rule, int search,
                      int gscale_given, float *gscale,
                      uint8_t *q, uint8_t *s_logical);

/* Quantization with the sparse residual lane ([TransFP4] §2.3 Eq.(3),
 * r = 1 per 32 values): res receives rows x cols/32 words (bf16 bits |
 * index << 16) of the largest-magnitude rotated value of every 32-value
 * unit, which is zeroed before the FP4 quantization (and before the NVFP4
 * tensor maximum).  Absmax block scales. */
int fp4o_quantize_residual(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                           int fmt, int block, int hadamard_k, int tie, int mx_rule,
                           int gscale_given, float *gscale, uint8_t *q, uint8_t *s_logical,
                           uint32_t *res);

/* Alternating refinement of the NVFP4 tensor scale (MSE group step, least-
 * squares global step), `rounds` evaluations from the absmax s_g; returns
 * the best s_g and its fp64 squared error (see the function's comment). */
int fp4o_nv_refine_gscale(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld,
                          int hadamard_k, int tie, int rounds, float *gscale, double *err);

/* Dequantization of the FP4 stream plus the residual lane, then the inverse
 * rotation. */
int fp4o_dequantize_residual(const uint8_t *q, const uint8_t *s_logical, float gscale,
                             const uint32_t *res, int64_t rows, int64_t cols, int fmt, int block,
                             int hadamard_k, float *out);

/* out: rows x cols fp32.  hadamard_k > 0 applies the (self-inverse)
 * rotation again to return to the original domain. */
int fp4o_dequantize(const uint8_t *q, const uint8_t *s_logical, float gscale,
                    int64_t rows, int64_t cols, int fmt, int block,
                    int hadamard_k, float *out);

/* MXFP4 scales (logical, rows x nkb, E8M0) -> NVFP4 scales (logical,
 * rows x 2*nkb, E4M3) and the tensor scale s_g = 2^E that keep every
 * element's dequantized value (see the function's comment). */
int fp4o_mx_scales_to_nv(const uint8_t *s_mx, int64_t rows, int64_t nkb, uint8_t *s_nv,
                         float *gscale);

/* INT4 group quantization (Table 5's INT4 baseline): per group of `group`
 * values, fp32 scale amax / 7 and codes round(x / s) in [-7, 7] (ties to
 * even); q is rows x cols int8, scales rows x cols/group fp32. */
int fp4o_int4_quantize_f32(const float *x, int64_t rows, int64_t cols, int group, int8_t *q,
                           float *scales);
int fp4o_int4_dequantize(const int8_t *q, const float *scales, int64_t rows, int64_t cols, int group,
                         float *out);

/* The TransFP4 method of the page's Table 5 on fp32 rows: H_k, the residual
 * lane (one value per 32), and per 32-value unit the better of an NVFP4 and
 * an INT4 candidate by squared error (see the function's comment).  out:
 * rows x cols fp32 reconstruction in the original domain; choice: rows x
 * cols/32 bytes, 0 = NVFP4, 1 = INT4. */
int fp4o_transfp4_f32(const float *x, int64_t rows, int64_t cols, int hadamard_k, int tie,
                      int allow_int4, float *out, uint8_t *choice);

/* logical scales (rows x nkb) -> tcgen05 scale-atom layout/* logical scales (rows x nkb) -> tcgen05 scale-atom layout
 * (pad128(rows) x pad4(nkb) bytes, padding bytes 0), and back. */
void fp4o_scales_to_atoms(const uint8_t *s_logical, int64_t rows, int64_t nkb,
                          uint8_t *s_atoms);
void fp4o_scales_from_atoms(const uint8_t *s_atoms, int64_t rows, int64_t nkb,
                            uint8_t *s_logical);

/* C[m][n] = sum_k a[m][k] * w[n][k] in fp64, and bound[m][n] =
 * sum_k |a[m][k]| * |w[n][k]|.  a: M x K, w: N x K fp32 (dequantized). */
void fp4o_gemm_ref(const float *a, const float *w, int64_t M, int64_t N,
                   int64_t K, double *c, double *bound);

/* Number of OpenMP threads the oracle's row loops use (1 without OpenMP). */
int fp4o_num_threads(void);

#ifdef __cplusplus
}
#endif
#endif
