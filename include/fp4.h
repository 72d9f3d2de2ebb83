/*
 * fp4.h — C ABI of the B200 (sm_100a) microscaling FP4 library.
 *
 * Formats (element E2M1 in every case):
 *   MXFP4  32-element blocks along K, one E8M0 (power-of-two) scale per block.
 *   NVFP4  16-element blocks along K, one unsigned E4M3 scale per block, and
 *          one FP32 tensor-level scale s_g.
 *   MXFP4_16  16-element blocks along K, one E8M0 scale per block: the
 *          microscaling form with block size G = 16 (TransFP4 §1.1 leaves G
 *          open) and the 16-element scale vector the block-scaled MMA also
 *          takes with E8M0 scales.  It keeps MXFP4's scale encoding at
 *          NVFP4's block size, so the two effects that tell MXFP4 and NVFP4
 *          apart can be taken one at a time.
 * Sources: "Portable FP4 quantization (TransFP4)" §1.1 Eq.(1)
 * (x^_i = s_g s_b Q_f(x_i / (s_g s_b))) and Table 1; "4.5 FP8 and
 * NVFP4/MXFP4" §3.1 (E2M1 magnitudes), §3.3 and §4.1 (scale formats, the
 * two-level NVFP4 dequantization); "FP4 quantization analysis: MXFP4 vs
 * NVFP4" §3.2.3 (block-diagonal Hadamard H_k, k in {16,32,64,128}) and §3.3
 * (fused rotation kernel, FP4-specific operand re-layout for the GEMM).
 *
 * Conventions for every call:
 *   - All pointers are DEVICE pointers unless the name says host.  The caller
 *     allocates and owns every buffer; the library never allocates or frees
 *     device memory and keeps no pointer after the call returns.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are asynchronous and stream-ordered; none synchronizes
 *     the host.
 *   - Shapes are validated on the host before any launch; an invalid call
 *     launches nothing and returns an error code.  Errors raised by a
 *     launch return FP4_ERR_CUDA; faults of an earlier asynchronous launch
 *     surface on a later call or synchronization.
 *   - Inputs must be finite.  Quantization axis = contraction axis = K, the
 *     contiguous (column) axis of a row-major rows x cols tensor.
 *
 * Layouts:
 *   Packed elements q: rows x cols/2 bytes, row stride cols/2; byte j of a
 *     row holds element 2j in bits [3:0] and element 2j+1 in bits [7:4];
 *     bit 3 of a nibble is the sign.
 *   Scales s: the tile layout the block-scaled tensor-core MMA reads.
 *     Logical scale S[r][kb] (kb = block index along K, nkb = cols/block)
 *     lives at byte
 *       ((r/128) * ceil(nkb/4) + kb/4) * 512 + (r%32)*16 + ((r%128)/32)*4 + kb%4
 *     i.e. 512-byte atoms of 128 rows x 4 scales.  Rows are padded to a
 *     multiple of 128 and scale columns to a multiple of 4; fp4_quantize
 *     writes every padding byte as 0.
 */
#ifndef FP4_H
#define FP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FP4_OK = 0,
    FP4_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad enum     */
    FP4_ERR_UNSUPPORTED = 2,   /* shape or format combination not provided  */
    FP4_ERR_ALIGNMENT = 3,     /* pointer or stride not aligned as required */
    FP4_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed      */
    FP4_ERR_TIMEOUT = 5        /* a kernel gave up a bounded wait           */
} fp4_status;

typedef enum { FP4_MXFP4 = 0, FP4_NVFP4 = 1, FP4_MXFP4_16 = 2 } fp4_fmt;

/* E2M1 tie rule at exact midpoints: even code (IEEE style, default) or the
 * larger magnitude (reproduces the gpt-oss article's worked example). */
typedef enum { FP4_ROUND_EVEN = 0, FP4_ROUND_AWAY = 1 } fp4_round;

/* MXFP4 shared exponent: CEIL = smallest e with amax <= 6*2^e (no element
 * clips; default); FLOOR = floor(log2 amax) - 2 (the OCP MX rule; values
 * between 6 and 8 times the scale saturate to 6). */
typedef enum { FP4_MX_SCALE_CEIL = 0, FP4_MX_SCALE_FLOOR = 1 } fp4_mx_scale_rule;

/* Block-scale method ("FP4 quantization analysis: MXFP4 vs NVFP4" §3.3:
 * kernels with the "MSE" and the "Abs-Max" method).  ABSMAX (default): the
 * scale from the block max (mx_scale_rule for MXFP4).  MSE (§3.2.1, scales
 * that minimise sum ||Y^_i - X_i||^2): each block tries a fixed window of
 * scales around the absmax one and keeps the one with the smallest fp32
 * squared reconstruction error, summed in a fixed pairwise order; of equal
 * ones the first tried.  Windows, in the order tried:
 *   MXFP4, MXFP4_16: e_c (the CEIL exponent), e_c - 1 (unless e_c = -127);
 *          mx_scale_rule is not used;
 *   NVFP4: t0 (the absmax E4M3 code), t0-2, t0-1, t0+1, ..., t0+6, within
 *          1 .. 0x7E.  The tensor scale s_g stays the absmax one.
 * fp4_quantize only; fp4_linear and fp4_gemm_quantized return
 * FP4_ERR_UNSUPPORTED for MSE. */
typedef enum { FP4_SCALE_ABSMAX = 0, FP4_SCALE_MSE = 1 } fp4_scale_search;

typedef enum { FP4_OUT_F32 = 0, FP4_OUT_BF16 = 1 } fp4_dtype;

typedef struct {
    int round;          /* fp4_round                                          */
    int mx_scale_rule;  /* fp4_mx_scale_rule                                  */
    int gscale_given;   /* NVFP4: 1 = *gscale holds s_g on entry (offline
                           scale); 0 = s_g is computed from the tensor.       */
    int scale_search;   /* fp4_scale_search                                   */
    int weights_static; /* fp4_linear, M <= 16: 1 = W, its scales and gW are
                           written by no kernel that may still be running when
                           the call's kernels start (weights prepared once and
                           read-only, as in inference).  The decode kernel then
                           streams W while the work before it in the stream
                           finishes; activations and C stay ordered after it.
                           0 (default): W is read only after that work.      */
} fp4_opts;

/* Human-readable name of a status code (static string). */
const char *fp4_status_string(fp4_status st);

/* Sizes of the packed-element and scale buffers for a rows x cols tensor.
 * q_bytes = rows*cols/2; s_bytes = pad128(rows) * pad4(cols/block).
 * Host-only; block must be 32 for MXFP4 and 16 for NVFP4 and MXFP4_16
 * (fmt = FP4_MXFP4 with block = 16 is taken as FP4_MXFP4_16, here and in
 * fp4_quantize, fp4_dequantize and their residual forms). */
fp4_status fp4_quantize_sizes(int64_t rows, int64_t cols, int fmt, int block,
                              size_t *q_bytes, size_t *s_bytes);

/*
 * fp4_quantize — microscaling quantization, TransFP4 Eq.(1), optionally after
 * the block-diagonal Hadamard rotation H_k (MR-GPTQ §3.2.3) of every
 * contiguous k-element chunk along K.
 *
 *   x       bf16 input, rows x cols, row stride ld_x elements.  16-byte
 *           aligned; ld_x a multiple of 8.
 *   fmt     FP4_MXFP4 (block 32), FP4_NVFP4 (block 16) or FP4_MXFP4_16
 *           (block 16).
 *   hadamard_k  0 (no rotation) or 16, 32, 64, 128; cols % k == 0.  The
 *           rotation is the normalised Sylvester Walsh-Hadamard transform
 *           (stages h = 1, 2, ..., k/2, then x RN(1/sqrt(k))) in fp32.
 *   opts    may be NULL (= round even, CEIL, s_g computed).
 *   q       output, packed elements (layout above), 16-byte aligned.
 *   s       output, scales in the tile layout above (padding written 0).
 *   gscale  NVFP4 only (ignored for the E8M0 formats, may be NULL): one
 *           device fp32.
 *           gscale_given: read as s_g.  Otherwise written with
 *           s_g = amax(|H_k x|) / (6*448), or 1 for an all-zero tensor.
 * cols must be a multiple of 32 (also for NVFP4).  rows == 0 is a no-op.
 * rows * cols / 32 must stay below 2^32 (FP4_ERR_UNSUPPORTED otherwise; the
 * bound is above what device memory holds as bf16); the same holds for
 * fp4_dequantize and for M * K in fp4_linear.
 */
fp4_status fp4_quantize(const void *x, int64_t rows, int64_t cols, int64_t ld_x,
                        int fmt, int block, int hadamard_k, const fp4_opts *opts,
                        uint8_t *q, uint8_t *s, float *gscale, void *stream);

/*
 * fp4_dequantize — x^ = s_g * s_b * q ("4.5 FP8 and NVFP4/MXFP4" §4.1; for
 * MXFP4 s_g = 1 and s_b = 2^(byte-127)), NVFP4 computed as
 * RN(RN(s_g*s_b) * q).  hadamard_k > 0 applies H_k again (it is its own
 * inverse) to return to the unrotated domain; 0 leaves values rotated.
 *   q, s, gscale   as produced by fp4_quantize (gscale ignored for MXFP4
 *                  and MXFP4_16).
 *   out_dtype      FP4_OUT_F32 or FP4_OUT_BF16 (round to nearest even).
 *   out            rows x cols, row stride cols, 16-byte aligned.
 */
fp4_status fp4_dequantize(const uint8_t *q, const uint8_t *s, const float *gscale,
                          int64_t rows, int64_t cols, int fmt, int block,
                          int hadamard_k, int out_dtype, void *out, void *stream);

/*
 * fp4_quantize_residual — fp4_quantize with the sparse residual lane of
 * "Portable FP4 quantization (TransFP4)" §2.3 Eq.(3), one value per 32:
 *   x^ = H^T Q_f(H x - P H x) + H^T P H x,
 * P selecting, in every 32-value unit of the rotated row H x, the value of
 * largest magnitude (the first of equal ones).  That value is zeroed before
 * the FP4 quantization (the NVFP4 tensor scale is that of the FP4 stream) and
 * kept in `res`: rows x cols/32 uint32 words, row-major, each holding the
 * value's bf16 bits (round to nearest even) in bits 15:0 and its index in the
 * unit in bits 20:16.  Other arguments as fp4_quantize; absmax scales only
 * (FP4_SCALE_MSE: FP4_ERR_UNSUPPORTED).  res 4-byte aligned.
 */
fp4_status fp4_quantize_residual(const void *x, int64_t rows, int64_t cols, int64_t ld_x,
                                 int fmt, int block, int hadamard_k, const fp4_opts *opts,
                                 uint8_t *q, uint8_t *s, float *gscale, uint32_t *res, void *stream);

/* fp4_dequantize_residual — the inverse: the FP4 stream dequantized, the
 * residual value added at its index in fp32, then H^T as in fp4_dequantize. */
fp4_status fp4_dequantize_residual(const uint8_t *q, const uint8_t *s, const float *gscale,
                                   const uint32_t *res, int64_t rows, int64_t cols, int fmt,
                                   int block, int hadamard_k, int out_dtype, void *out, void *stream);

/* Bytes of scratch fp4_gemm needs for this shape (0 when none). Host-only. */
fp4_status fp4_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int fmt,
                                   size_t *bytes);

/*
 * fp4_gemm — W4A4 linear C = alpha * A W^T with FP32 accumulation
 * ("4.5 FP8 and NVFP4/MXFP4" §5: both operands in FP4 on the Blackwell
 * tensor cores), A: M x K, W: N x K, both quantized along K in the same
 * format by fp4_quantize (Aq/As, Wq/Ws).  alpha = s_gA * s_gW for NVFP4
 * (gA, gW device fp32), 1 for MXFP4 and MXFP4_16 (gA, gW ignored).
 *   K          multiple of 32 ("Portable FP4 quantization (TransFP4)" Table 3:
 *              the GEMM's K alignment is 32).  The tensor cores step K by
 *              256 per stage; the last step of a tail multiplies zeros read
 *              past K with the zero padding scales fp4_quantize writes.
 *   out_dtype  FP4_OUT_F32 or FP4_OUT_BF16.  C row-major, row stride ldc
 *              elements (ldc >= N).
 *   workspace  device scratch of at least fp4_gemm_workspace_size() bytes
 *              (may be NULL when that size is 0).
 * Rotated operands: quantize both A and W with the same hadamard_k;
 * (X H)(W H)^T = X W^T, so C needs no correction.
 * M <= 16 runs the decode (weight-streaming, split-K) kernel; larger M the
 * tiled tensor-core kernel.  M, N and K above 2^30 return FP4_ERR_UNSUPPORTED
 * (also from the workspace-size queries and fp4_linear).
 */
fp4_status fp4_gemm(const uint8_t *Aq, const uint8_t *As, const float *gA,
                    const uint8_t *Wq, const uint8_t *Ws, const float *gW,
                    int64_t M, int64_t N, int64_t K, int fmt, int out_dtype,
                    void *C, int64_t ldc, void *workspace, size_t ws_bytes,
                    void *stream);

/*
 * fp4_gemm_quantized — the product of fp4_gemm, C = alpha * A W^T with FP32
 * accumulation, quantized again along N in the tensor-core kernel's epilogue
 * for the next layer, which then takes C as its activations: the "custom
 * epilogue fusing quantization and scale computation" that "FP4
 * quantization analysis: MXFP4 vs NVFP4" §3.3 describes for QuTLASS, with
 * the per-unit encoding of fp4_quantize (TransFP4 §1.1 Eq.(1)) applied to
 * the FP32 values alpha * acc.
 *   Aq/As/gA, Wq/Ws/gW, fmt   as for fp4_gemm.
 *   out_fmt   FP4_MXFP4 or FP4_NVFP4 (may differ from fmt; FP4_MXFP4_16
 *             output: FP4_ERR_UNSUPPORTED).
 *   opts      round and mx_scale_rule as for fp4_quantize; may be NULL.
 *   gC        NVFP4 output: the tensor scale s_g of C, one device fp32, given
 *             (a whole-tensor maximum is not known until every tile is done,
 *             so it is not computed here).  Ignored for MXFP4.
 *   Cq        output, M x N/2 bytes of packed elements, 16-byte aligned.
 *   Cs        output, the scales in the tile layout of fp4_quantize
 *             (fp4_quantize_sizes(M, N, out_fmt, ...) bytes; the padding rows
 *             are written 0), 16-byte aligned.
 * Shapes: M > 16 (the tiled kernel), K multiple of 32, N multiple of 128;
 * otherwise FP4_ERR_UNSUPPORTED with nothing launched.  Each 32-element unit
 * is encoded as fp4_quantize encodes one, from the FP32 values fp4_gemm
 * returns with FP4_OUT_F32 for the same operands.
 */
fp4_status fp4_gemm_quantized(const uint8_t *Aq, const uint8_t *As, const float *gA,
                              const uint8_t *Wq, const uint8_t *Ws, const float *gW,
                              int64_t M, int64_t N, int64_t K, int fmt, int out_fmt,
                              const fp4_opts *opts, const float *gC, uint8_t *Cq,
                              uint8_t *Cs, void *stream);


/*
 * fp4_nv_refine_gscale — the NVFP4 tensor scale s_g refined by alternating
 * group and global steps ("FP4 quantization analysis: MXFP4 vs NVFP4"
 * §3.2.1), for an offline (weight) quantization that then runs
 * fp4_quantize with scale_search = FP4_SCALE_MSE and gscale_given = 1.
 * From the absmax s_g, each of `rounds` rounds (1..64) quantizes x (with
 * H_k when hadamard_k > 0) by the MSE block-scale search under the current
 * s_g, measures E = sum (x_i - y_i)^2 over the rotated values and their
 * reconstructions, and moves s_g to the least-squares scale of the chosen
 * codes, sum x_i u_i / sum u_i^2 with u_i = s_b q_i (kept if that is 0 or
 * not a positive finite float).  *gscale receives the evaluated s_g with the
 * smallest E (the first of equal ones; rounds = 1 gives the absmax s_g).
 * Sums are fp64 in a fixed order (a unit's 32 values, a row's units, the
 * rows), so the result is reproducible.
 *   x, rows, cols, ld_x, hadamard_k, opts (round)   as fp4_quantize.
 *   q, s       scratch of fp4_quantize_sizes(rows, cols, FP4_NVFP4, 16)
 *              bytes; they end holding the last round's quantization.
 *   workspace  fp4_nv_refine_gscale_workspace_size() bytes, 256-byte
 *              aligned.
 *   gscale     output, one device fp32.
 * About 5 launches per round; meant to run once per weight.
 */
fp4_status fp4_nv_refine_gscale_workspace_size(int64_t rows, int64_t cols, size_t *bytes);
fp4_status fp4_nv_refine_gscale(const void *x, int64_t rows, int64_t cols, int64_t ld_x,
                                int hadamard_k, const fp4_opts *opts, int rounds, uint8_t *q,
                                uint8_t *s, void *workspace, size_t ws_bytes, float *gscale,
                                void *stream);

/*
 * fp4_mx_to_nv_scales — late binding of an MXFP4 tensor to the NVFP4 scale
 * form ("Portable FP4 quantization (TransFP4)" §2.5, §3.4), so that NVFP4
 * activations can meet MXFP4 weights in the NVFP4 tensor-core product
 * (fp4_linear / fp4_gemm with fmt = FP4_NVFP4 and the same packed elements).
 * Each 32-block scale 2^e becomes two 16-block E4M3 scales 2^(e - E) under
 * the tensor scale s_g = 2^E, E = max(e_max - 8, -126) (e_max: the largest
 * block exponent), so s_g * s_b = 2^e and every element dequantizes to the
 * same value.  Blocks more than 17 binades below the largest take the E4M3
 * rounding of 2^(e - E), which is 0 from 2^-10 down; E8M0 NaN becomes E4M3
 * NaN.  Three small launches; meant to run once per weight.
 *   s_mx    MXFP4 (32-element block) scales of a rows x cols tensor in the
 *           tile layout, as
 *           fp4_quantize writes them (cols multiple of 32).
 *   s_nv    output: fp4_quantize_sizes(rows, cols, FP4_NVFP4, 16) scale
 *           bytes in the tile layout, padding written 0.
 *   gscale  output: s_g, one device fp32 (4-byte aligned).
 */
fp4_status fp4_mx_to_nv_scales(const uint8_t *s_mx, int64_t rows, int64_t cols, uint8_t *s_nv,
                               float *gscale, void *stream);

/* Bytes of device scratch fp4_linear needs (quantized activations, their
 * scales and tensor scale, and the GEMM workspace).  Host-only. */
fp4_status fp4_linear_workspace_size(int64_t M, int64_t N, int64_t K, int fmt, size_t *bytes);

/*
 * fp4_linear — the W4A4 linear layer from bf16 activations: x (M x K bf16,
 * row stride ld_x) is quantized online ("4.5 FP8 and NVFP4/MXFP4" §4.2:
 * online quantization from BF16 needs no calibration data) in the weight's
 * format, optionally rotated by H_k ("FP4 quantization analysis" §3.2.3:
 * activations rotated online, weights rotated offline — W must have been
 * quantized with the same hadamard_k), then C = alpha * x_q W_q^T as in
 * fp4_gemm.  M <= 16 is the decode case the weight stream dominates: one
 * kernel launch, whose warps quantize each 256-wide K step of x straight
 * into the pipeline stage the tensor cores read (bit-identical to
 * fp4_quantize + fp4_gemm with the same work split).  Splits that cut tiles
 * between CTAs outside a cluster (very few or very many 128-row W tiles)
 * take two launches: the activation quantizer, then fp4_gemm's kernel.
 *   gA      NVFP4 activation tensor scale: NULL = computed from x (dynamic),
 *           else a device fp32 holding a static s_g.  Ignored for MXFP4 and
 *           MXFP4_16.
 *   opts    rounding options for the activation quantization (may be NULL;
 *           gscale_given is ignored, gA decides).
 *   workspace  at least fp4_linear_workspace_size() bytes, 256-byte aligned;
 *           its contents on entry do not matter.
 */
fp4_status fp4_linear(const void *x, int64_t M, int64_t K, int64_t ld_x, int fmt, int hadamard_k,
                      const fp4_opts *opts, const float *gA, const uint8_t *Wq, const uint8_t *Ws,
                      const float *gW, int64_t N, int out_dtype, void *C, int64_t ldc,
                      void *workspace, size_t ws_bytes, void *stream);

/*
 * fp4_linear_residual — fp4_linear for the decode case (M <= 16) with the
 * sparse residual lane of "Portable FP4 quantization (TransFP4)" §2.3
 * Eq.(3) in the activations: with x rotated by H_k (hadamard_k, as W was),
 *   C = alpha * Q_f(H x - P H x) W_q^T  +  (P H x) W_q^T,
 * where P keeps, in every 32-value unit of each rotated activation row, the
 * value of largest magnitude (the first of equal ones) rounded to bf16, as
 * fp4_quantize_residual defines it; the FP4 stream's NVFP4 tensor scale is
 * that of the values left (computed, or the static gA).  One launch: the
 * lane's product runs on the tensor cores with the activations', each
 * residual split into terms the block-scaled product represents exactly:
 * 4 terms under E8M0 scales for MXFP4 and MXFP4_16 (every bf16 value of
 * magnitude >= 2^-126), 2 terms under E4M3 scales and one of two
 * power-of-two scales per activation row, 2^10 apart, for NVFP4 (exact for
 * residuals within a factor 2^19 of their row's largest; smaller ones are
 * rounded at that row's finest E4M3 step).
 *   Arguments as fp4_linear, without a workspace (none is needed): W is the
 *   weight as fp4_quantize wrote it (with the same hadamard_k).  M > 16
 *   returns FP4_ERR_UNSUPPORTED, as does FP4_SCALE_MSE.
 */
fp4_status fp4_linear_residual(const void *x, int64_t M, int64_t K, int64_t ld_x, int fmt, int hadamard_k,
                               const fp4_opts *opts, const float *gA, const uint8_t *Wq, const uint8_t *Ws,
                               const float *gW, int64_t N, int out_dtype, void *C, int64_t ldc, void *stream);

/*
 * fp4_gemm_decode_noalloc — the decode product of fp4_gemm (M <= 16) for
 * callers that cannot allocate device memory at call time (inside a stream
 * capture that must not add allocations, a plugin given fixed buffers, a
 * process with a fixed memory budget).  It has no counterpart on the source
 * pages: it is the same computation as fp4_gemm, with the split-K partials
 * kept in a 4 MiB array inside this library instead of a caller workspace.
 *   Arguments as fp4_gemm, without workspace.  M must be <= 16 and
 *   fp4_gemm_workspace_size(M, N, K, fmt) must be <= 4 MiB, else
 *   FP4_ERR_UNSUPPORTED (nothing launched).
 *   The array is a device variable: every GPU that loads the library holds
 *   4 MiB for it until the process exits.  The first call on a device looks
 *   up the array's device address (with that device current) and keeps it
 *   for the life of the process; make that first call before any stream
 *   capture.  A cudaDeviceReset (or any other teardown of the device's
 *   primary context) makes the kept address stale: after one, this entry
 *   point must not be called again in the same process.  All calls share the array: calls whose
 *   kernels overlap on the GPU (different streams without ordering) race and
 *   give wrong results.  Nothing in it needs to start at zero; it keeps the
 *   last call's partial sums.
 * Allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 */
fp4_status fp4_gemm_decode_noalloc(const uint8_t *Aq, const uint8_t *As, const float *gA,
                                   const uint8_t *Wq, const uint8_t *Ws, const float *gW,
                                   int64_t M, int64_t N, int64_t K, int fmt, int out_dtype,
                                   void *C, int64_t ldc, void *stream);

/* Number of kernels this library has launched in this process so far
 * (host-side counter; diagnostics and launch accounting). */
uint64_t fp4_kernel_launches(void);

/* Failure-detection test hook: for tests only, not for production use, and
 * not thread-safe.  The setting is one process-wide value that the next GEMM
 * launch from any host thread consumes, so use it only while a single thread
 * launches GEMMs.  With stall != 0 the next GEMM launch
 * (fp4_gemm, fp4_gemm_quantized, fp4_linear or fp4_gemm_decode_noalloc)
 * issues no operand loads,
 * so its MMA warp's bounded wait gives up after budget_ns nanoseconds
 * (0 = the default of 2 s): the kernel sets the device error word, stores
 * nothing, frees its tensor memory and returns, and fp4_check_device_status()
 * then reports FP4_ERR_TIMEOUT.  The context stays usable.  A nonzero
 * budget_ns with stall == 0 only shortens the waits of the next launch.
 * Host-side, applies to one launch.  fp4_linear_residual is a GEMM launch too. */
fp4_status fp4_test_inject_stall(int stall, uint64_t budget_ns);

/* Reads and clears the device-side error word that kernels set when a
 * bounded wait gives up.  Synchronizes `stream`.  Returns FP4_ERR_TIMEOUT if
 * it was set, else FP4_OK (or FP4_ERR_CUDA). */
fp4_status fp4_check_device_status(void *stream);

#ifdef __cplusplus
}
#endif
#endif
