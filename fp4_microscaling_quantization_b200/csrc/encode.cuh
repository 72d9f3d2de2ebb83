// encode.cuh — the per-unit arithmetic of FP4 quantization, shared by the
// streaming quantize kernels and the decode GEMM's fused activation
// quantizer so both produce the same bits.
//
// Method: "Portable FP4 quantization (TransFP4)" §1.1 Eq.(1) with absmax
// block scales and nearest rounding; the NVFP4 two-level scale ("4.5 FP8 and
// NVFP4/MXFP4" §4.1); the block-diagonal Hadamard rotation H_k ("FP4
// quantization analysis: MXFP4 vs NVFP4" §3.2.3).  A unit is 32 consecutive
// elements of a row: one MXFP4 block, or two 16-element blocks (NVFP4, or
// MXFP4 on 16-element blocks: E8M0 scales at NVFP4's block size).
#pragma once

#include "common.cuh"

namespace fp4 {

// bf16 pairs -> 32 fp32 values.
FP4_DEV void unpack_unit(const uint4 *raw, float *v)
{
#pragma unroll
    for (int c = 0; c < 4; c++) {
        const uint4 w = raw[c];
        v[8 * c + 0] = bf16lo(w.x);
        v[8 * c + 1] = bf16hi(w.x);
        v[8 * c + 2] = bf16lo(w.y);
        v[8 * c + 3] = bf16hi(w.y);
        v[8 * c + 4] = bf16lo(w.z);
        v[8 * c + 5] = bf16hi(w.z);
        v[8 * c + 6] = bf16lo(w.w);
        v[8 * c + 7] = bf16hi(w.w);
    }
}

// Two-wide fp32 arithmetic (sm_100's packed f32x2 add, sub and multiply):
// each half is rounded to nearest even exactly as the scalar operation, and
// subnormals are kept (no .ftz), so results are those of two __fadd_rn /
// __fsub_rn / __fmul_rn calls, in half the instructions (checked on the B200
// over random operands of every class).  One hazard: ptxas contracts a packed
// product that feeds a packed sum or difference into a fused multiply-add
// (CUDA 12.9, sm_100a, in spite of .rn and -fmad=false), which skips the
// product's rounding.  So no packed product here feeds an add or subtract:
// the packed multiplies come last (the rotation's c_k, the block scales),
// and sums of products stay scalar.
// (a0, a1), (b0, b1) -> (a0 + b0, a1 + b1), (a0 - b0, a1 - b1)
FP4_DEV void add_sub_x2(float &a0, float &a1, float &b0, float &b1)
{
    asm("{\n\t.reg .b64 pa, pb, ps, pd;\n\t"
        "mov.b64 pa, {%0, %1};\n\tmov.b64 pb, {%2, %3};\n\t"
        "add.rn.f32x2 ps, pa, pb;\n\tsub.rn.f32x2 pd, pa, pb;\n\t"
        "mov.b64 {%0, %1}, ps;\n\tmov.b64 {%2, %3}, pd;\n\t}"
        : "+f"(a0), "+f"(a1), "+f"(b0), "+f"(b1));
}

// (a0, a1) *= (m0, m1)
FP4_DEV void mul_x2(float &a0, float &a1, float m0, float m1)
{
    asm("{\n\t.reg .b64 pa, pm;\n\t"
        "mov.b64 pa, {%0, %1};\n\tmov.b64 pm, {%2, %3};\n\t"
        "mul.rn.f32x2 pa, pa, pm;\n\tmov.b64 {%0, %1}, pa;\n\t}"
        : "+f"(a0), "+f"(a1)
        : "f"(m0), "f"(m1));
}

// (a0, a1) = (a0 * m0 + c0, a1 * m1 + c1), each rounded once (fused)
FP4_DEV void fma_x2(float &a0, float &a1, float m0, float m1, float c0, float c1)
{
    asm("{\n\t.reg .b64 pa, pm, pc;\n\t"
        "mov.b64 pa, {%0, %1};\n\tmov.b64 pm, {%2, %3};\n\tmov.b64 pc, {%4, %5};\n\t"
        "fma.rn.f32x2 pa, pa, pm, pc;\n\tmov.b64 {%0, %1}, pa;\n\t}"
        : "+f"(a0), "+f"(a1)
        : "f"(m0), "f"(m1), "f"(c0), "f"(c1));
}

// v[j] *= m0 and v[j + 16] *= m1 for j < 16: the two 16-element halves of a
// unit (one scale each for 16-element blocks; m0 = m1 for one scale).
FP4_DEV void scale_halves(float *v, float m0, float m1)
{
#pragma unroll
    for (int j = 0; j < 16; j++) mul_x2(v[j], v[j + 16], m0, m1);
}

// Normalised Sylvester Walsh-Hadamard transform of every k-chunk, stages
// h = 1, 2, ..., k/2 in ascending order: (a, b) -> (a + b, a - b) with a the
// element whose index has bit h clear; then every value times ck.  Stages
// with h >= 32 pair this lane with lane ^ (h / 32).  Stages h < 16 run two
// butterflies per instruction, one in each 16-element half of the unit
// (elements j and j + 16 share a packed operand).
template <int HK>
FP4_DEV void fwht_unit(float *v, float ck, int lane)
{
#pragma unroll
    for (int h = 1; h < (HK < 16 ? HK : 16); h <<= 1) {
#pragma unroll
        for (int j = 0; j < 16; j++) {
            if (j & h) continue;
            add_sub_x2(v[j], v[j + 16], v[j + h], v[j + h + 16]);
        }
    }
    if (HK >= 32) {
#pragma unroll
        for (int j = 0; j < 16; j++) {
            const float a = v[j], b = v[j + 16];
            v[j] = __fadd_rn(a, b);
            v[j + 16] = __fsub_rn(a, b);
        }
    }
#pragma unroll
    for (int lm = 1; lm < HK / 32; lm <<= 1) {
        // lower lane: b + a; upper lane: a - b = (-1) * b + a.  One fused
        // multiply-add with a lane's sign s = +-1: the product v * s is exact,
        // so v * s + o rounds once to the same sum as o + (+-v), two elements
        // per instruction, without a select or a sign flip per value.
        const float s = (lane & lm) ? -1.0f : 1.0f;
#pragma unroll
        for (int j = 0; j < 16; j++) {
            const float o0 = __shfl_xor_sync(0xFFFFFFFFu, v[j], lm);
            const float o1 = __shfl_xor_sync(0xFFFFFFFFu, v[j + 16], lm);
            fma_x2(v[j], v[j + 16], s, s, o0, o1);
        }
    }
    scale_halves(v, ck, ck);
}

FP4_DEV float nv_global_from_amax(float amax)
{
    return (amax > 0.0f && amax <= kFltMax) ? __fdiv_rn(amax, 2688.0f) : 1.0f;
}

// Largest |v_i| of N consecutive values, as a balanced tree of pairwise
// maxima: the maximum is exact and independent of order, so this equals a
// running maximum, with a dependency chain of log2 N steps instead of N.
template <int N>
FP4_DEV float absmax_tree(const float *v)
{
    float t[N / 2];
#pragma unroll
    for (int i = 0; i < N / 2; i++) t[i] = fmaxf(fabsf(v[2 * i]), fabsf(v[2 * i + 1]));
#pragma unroll
    for (int w = N / 4; w >= 1; w >>= 1) {
#pragma unroll
        for (int i = 0; i < w; i++) t[i] = fmaxf(t[i], t[i + w]);
    }
    return t[0];
}

// Sparse residual lane ("Portable FP4 quantization (TransFP4)" §2.3 Eq.(3),
// one value per 32): the value of largest magnitude in the rotated unit v
// (the first of equal ones) leaves the FP4 stream: it is zeroed in v and
// returned as a word holding its bf16 rounding (RNE) and its index << 16.
FP4_DEV uint32_t extract_residual(float *v)
{
    // the maximum by a balanced tree, then the first index that reaches it:
    // a short dependency chain instead of a 32-step running search
    const float amax = absmax_tree<32>(v);
    uint32_t hit = 0;
#pragma unroll
    for (int i = 0; i < 32; i++) hit |= (fabsf(v[i]) == amax ? 1u : 0u) << i;
    const int best = __ffs(hit) - 1;
    float top = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; i++) {
        if (i == best) {
            top = v[i];
            v[i] = 0.0f;
        }
    }
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(top)) | ((uint32_t)best << 16);
}

// NVFP4 encode factor of a block scale with decode factor d: RN(1/d),
// clamped to the largest float; 0 for d = 0 (the block encodes as zeros).
FP4_DEV float nv_encode_factor(float d) { return (d == 0.0f) ? 0.0f : fminf(__frcp_rn(d), kFltMax); }

// Per-CTA tables of the NVFP4 block scales under one tensor scale s_g: the
// decode factor d = RN(s_g * s_b) and the encode factor RN(1/d) of every
// E4M3 code 0 .. 0x7E, so that a block looks them up instead of converting
// its code and dividing (the same values, computed once per CTA).
struct NvScaleTables {
    float d[128];
    float r[128];
};

// Fills the tables (any number of threads; the caller synchronises).
FP4_DEV void nv_tables_fill(NvScaleTables &t, float sg, int tid, int nthreads)
{
    for (int c = tid; c < 128; c += nthreads) {
        const float d = (c < 0x7F) ? __fmul_rn(sg, e4m3_to_f32((uint32_t)c)) : 0.0f;
        t.d[c] = d;
        t.r[c] = nv_encode_factor(d);
    }
}

// E2M1 codes of 32 values already divided by their block scale, packed as
// 16 bytes of nibbles (even element in the low nibble).
FP4_DEV void e2m1_pack_unit(const float *v, int round_away, uint4 &out)
{
    if (!round_away) {
        out.x = e2m1x8_rn(v + 0);
        out.y = e2m1x8_rn(v + 8);
        out.z = e2m1x8_rn(v + 16);
        out.w = e2m1x8_rn(v + 24);
    } else {
        out.x = e2m1x8_away(v + 0);
        out.y = e2m1x8_away(v + 8);
        out.z = e2m1x8_away(v + 16);
        out.w = e2m1x8_away(v + 24);
    }
}

// Scale and element encoding of one rotated 32-element unit (TransFP4
// Eq.(1): MXFP4 power-of-two scale; NVFP4 E4M3 block scale under the tensor
// scale sg).  v is scaled in place; the 32 E2M1 codes come back as 16 bytes
// of nibbles (even element in the low nibble) and the return value holds the
// scale byte (MXFP4) or the two block-scale bytes, first block low (NVFP4,
// MXFP4_16).
template <int FMT>
FP4_DEV uint32_t encode_unit(float *v, float sg, float six_sg, int round_away, int mx_floor, uint4 &out,
                             const NvScaleTables *tab = nullptr)
{
    uint32_t sbytes;
    if (FMT == FP4_MXFP4) {
        const float amax = absmax_tree<32>(v);
        const int e = mx_exponent(amax, mx_floor);
        const float inv = exp2i(-e);
        scale_halves(v, inv, inv);
        sbytes = (uint32_t)(e + 127);
    } else if (FMT == FP4_MXFP4_16) {
        const int e0 = mx_exponent(absmax_tree<16>(v), mx_floor);
        const int e1 = mx_exponent(absmax_tree<16>(v + 16), mx_floor);
        scale_halves(v, exp2i(-e0), exp2i(-e1));
        sbytes = (uint32_t)(e0 + 127) | ((uint32_t)(e1 + 127) << 8);
    } else {
        float r[2];
        sbytes = 0;
#pragma unroll
        for (int b = 0; b < 2; b++) {
            const float amax = absmax_tree<16>(v + 16 * b);
            const uint32_t sb = e4m3_rn(__fdiv_rn(amax, six_sg));
            r[b] = tab ? tab->r[sb] : nv_encode_factor(__fmul_rn(sg, e4m3_to_f32(sb)));
            sbytes |= sb << (8 * b);
        }
        scale_halves(v, r[0], r[1]);
    }
    e2m1_pack_unit(v, round_away, out);
    return sbytes;
}

// ---- the "MSE" scale method ------------------------------------------------
// "FP4 quantization analysis: MXFP4 vs NVFP4" §3.2.1 (block scales chosen to
// minimise sum ||Y^_i - X_i||^2) and §3.3 (quantization kernels with the MSE
// and the Abs-Max method).  Each block tries a fixed window of scales around
// its absmax scale and keeps the one whose reconstruction has the smallest
// squared error; of equal ones the first tried.

// The E2M1 grid value nearest to a >= 0 (saturating at 6), ties as the
// encoder breaks them: the magnitude the hardware conversion's code decodes
// to, computed in fp32 without a conversion.  The grid step is 1/2 below 2,
// 1 up to 4 and 2 from 4 to 6.  Adding and then subtracting M = 1.5 * 2^22,
// 2^23 or 2^24 rounds a to a multiple of that step, ties to even (a + M lies
// in the binade whose ulp is the step; the subtraction is exact); the even
// multiple is the even code in every step.  Magnitudes past 6 saturate.
// Ties away: a value exactly half a step above its even rounding goes up.
FP4_DEV float e2m1_grid_magnitude(float a, int round_away)
{
    const bool lo = a < 2.0f, mid = a < 4.0f;
    const float m = lo ? 6291456.0f : (mid ? 12582912.0f : 25165824.0f);
    float r = __fsub_rn(__fadd_rn(a, m), m);
    if (round_away) {
        const float h = lo ? 0.25f : (mid ? 0.5f : 1.0f);
        if (__fsub_rn(a, r) == h) r = __fadd_rn(r, __fadd_rn(h, h));
    }
    return fminf(r, 6.0f);
}

// Squared reconstruction error of N values x under the block scale with
// decode factor d and encode factor r (x_i * r is what the encoder rounds):
// y_i = RN(q_i * d), e_i = RN(x_i - y_i), each e_i^2 rounded, then summed
// as a fixed pairwise tree: adjacent pairs first, then the first half of
// the partial sums plus the second half until one value remains.  Computed
// on magnitudes: y_i has the sign of x_i (r, d > 0) and rounding is
// symmetric, so RN(|x_i| - |y_i|) is e_i up to its sign and squares alike.
template <int N>
FP4_DEV float block_sq_error(const float *x, float r, float d, int round_away)
{
    float t[N / 2];
#pragma unroll
    for (int i = 0; i < N / 2; i++) {
        // scalar: a packed product here would be contracted into the
        // following subtraction (see add_sub_x2)
        const float a0 = fabsf(x[2 * i]), a1 = fabsf(x[2 * i + 1]);
        const float y0 = __fmul_rn(e2m1_grid_magnitude(__fmul_rn(a0, r), round_away), d);
        const float y1 = __fmul_rn(e2m1_grid_magnitude(__fmul_rn(a1, r), round_away), d);
        const float e0 = __fsub_rn(a0, y0);
        const float e1 = __fsub_rn(a1, y1);
        t[i] = __fadd_rn(__fmul_rn(e0, e0), __fmul_rn(e1, e1));
    }
#pragma unroll
    for (int w = N / 4; w >= 1; w >>= 1) {
#pragma unroll
        for (int i = 0; i < w; i++) t[i] = __fadd_rn(t[i], t[i + w]);
    }
    return t[0];
}

// The MSE choice between the CEIL exponent e of an E8M0-scaled block of N
// values and e - 1 (not below -127): e - 1 only if its error is smaller.
template <int N>
FP4_DEV int mx_mse_exponent(const float *x, int round_away)
{
    int e = mx_exponent(absmax_tree<N>(x), 0);
    if (e > -127) {
        const float e0 = block_sq_error<N>(x, exp2i(-e), exp2i(e), round_away);
        const float e1 = block_sq_error<N>(x, exp2i(1 - e), exp2i(e - 1), round_away);
        if (e1 < e0) e -= 1;
    }
    return e;
}

// encode_unit with the MSE method.  Candidates, in the order tried:
//   MXFP4, MXFP4_16: e_c (the CEIL exponent), then e_c - 1 unless
//          e_c = -127; the FLOOR rule's exponent is always one of the two.
//   NVFP4: t0 (the absmax E4M3 code), then t0 - 2, t0 - 1, t0 + 1 .. t0 + 6,
//          each only within 1 .. 0x7E: scales that put the block max between
//          about 3.6 and 7.3 on the grid.  Decode and encode factors come
//          from `tab`.
template <int FMT>
FP4_DEV uint32_t encode_unit_mse(float *v, float six_sg, int round_away, const NvScaleTables *tab, uint4 &out)
{
    uint32_t sbytes;
    if (FMT == FP4_MXFP4) {
        const int e = mx_mse_exponent<32>(v, round_away);
        const float inv = exp2i(-e);
        scale_halves(v, inv, inv);
        sbytes = (uint32_t)(e + 127);
    } else if (FMT == FP4_MXFP4_16) {
        const int e0 = mx_mse_exponent<16>(v, round_away);
        const int e1 = mx_mse_exponent<16>(v + 16, round_away);
        scale_halves(v, exp2i(-e0), exp2i(-e1));
        sbytes = (uint32_t)(e0 + 127) | ((uint32_t)(e1 + 127) << 8);
    } else {
        sbytes = 0;
#pragma unroll
        for (int b = 0; b < 2; b++) {
            float *x = v + 16 * b;
            const int t0 = (int)e4m3_rn(__fdiv_rn(absmax_tree<16>(x), six_sg));
            int best = t0;
            float best_err = block_sq_error<16>(x, tab->r[t0], tab->d[t0], round_away);
#pragma unroll 1
            for (int j = -2; j <= 6; j++) {
                const int c = t0 + j;
                if (j == 0 || c < 1 || c > 0x7E) continue;
                const float err = block_sq_error<16>(x, tab->r[c], tab->d[c], round_away);
                if (err < best_err) {
                    best = c;
                    best_err = err;
                }
            }
            sbytes |= (uint32_t)best << (8 * b);
        }
        scale_halves(v, tab->r[sbytes & 0xFF], tab->r[sbytes >> 8]);
    }
    e2m1_pack_unit(v, round_away, out);
    return sbytes;
}

}  // namespace fp4
