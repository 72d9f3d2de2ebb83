// common.cuh — device helpers shared by the sm_100a kernels of this library.
//
// Number formats ("4.5 FP8 and NVFP4/MXFP4", §1.2, §3.1, §3.3):
//   E2M1 element: 1 sign / 2 exponent / 1 mantissa bit, magnitudes
//   {0, 0.5, 1, 1.5, 2, 3, 4, 6};  E4M3 scale: bias 7, max 448, NaN only;
//   E8M0 scale: 2^(byte - 127).
// Conversions use the sm_100a hardware converters (round to nearest even,
// saturating to the largest finite value); every fp32 arithmetic step is an
// explicit round-to-nearest intrinsic so that no multiply-add is contracted.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "../../include/fp4.h"

#define FP4_DEV __device__ __forceinline__

namespace fp4 {

// Host-side launch accounting (fp4_kernel_launches).
void count_launches(int n);

// Launches `kern` on `st`; with `pdl` the launch may overlap the tail of the
// previous kernel in the stream (programmatic stream serialization).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                            Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    count_launches(1);
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

constexpr float kFltMax = 3.40282346638528859812e+38f;

// ---- division by a launch-invariant divisor ---------------------------------
// q = floor(n / d) for 32-bit unsigned n and d >= 1 by one high multiply, a
// subtract and two shifts: the round-up multiplier with one extra bit of
// Granlund and Montgomery, "Division by Invariant Integers using
// Multiplication" (PLDI 1994), section 4:
//   l = ceil(log2 d),  m = floor(2^32 (2^l - d) / d) + 1,
//   t = mulhi(m, n),   q = (t + ((n - t) >> min(l, 1))) >> max(l - 1, 0).
// Exact for every n < 2^32.  The kernels use it for the row of a 32-element
// unit (unit index / units per row), which a 64-bit division made the largest
// integer cost of the streaming kernels.
struct FastDiv {
    uint32_t d, m, s1, s2;
};

inline FastDiv make_fastdiv(uint32_t d)
{
    uint32_t l = 0;
    while ((1ull << l) < (uint64_t)d) l++;
    FastDiv f;
    f.d = d;
    f.m = (uint32_t)(((1ull << 32) * ((1ull << l) - (uint64_t)d)) / d + 1);
    f.s1 = l > 0 ? 1u : 0u;
    f.s2 = l > 0 ? l - 1 : 0u;
    return f;
}

FP4_DEV uint32_t fastdiv(uint32_t n, const FastDiv &f)
{
    const uint32_t t = __umulhi(n, f.m);
    return (t + ((n - t) >> f.s1)) >> f.s2;
}

// ---- programmatic dependent launch -----------------------------------------
// A kernel launched with programmatic stream serialization may start before
// its predecessor in the stream has finished; it must call grid_dep_wait()
// before reading anything the predecessor wrote (or writing anything it
// reads).  Both are no-ops for ordinary launches.
FP4_DEV void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
FP4_DEV void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---- bf16 -----------------------------------------------------------------
// Two bf16 values packed in a 32-bit word -> fp32 (exact).
FP4_DEV float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
FP4_DEV float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ---- E2M1 -------------------------------------------------------------------
// Eight fp32 values -> eight E2M1 codes (round to nearest even, saturate at
// +-6), value i in bits [4i+3 : 4i].
FP4_DEV uint32_t e2m1x8_rn(const float *v)
{
    uint32_t r;
    asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
        "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
        : "=r"(r)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return r;
}

// Nearest E2M1 code with midpoints going to the larger magnitude: the code
// is the number of midpoints 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5 that |v|
// reaches; the sign bit is copied from v.
FP4_DEV uint32_t e2m1_away(float v)
{
    float a = fabsf(v);
    uint32_t c = (a >= 0.25f) + (a >= 0.75f) + (a >= 1.25f) + (a >= 1.75f) + (a >= 2.5f) +
                 (a >= 3.5f) + (a >= 5.0f);
    return c | ((__float_as_uint(v) >> 28) & 8u);
}

FP4_DEV uint32_t e2m1x8_away(const float *v)
{
    uint32_t r = 0;
#pragma unroll
    for (int i = 0; i < 8; i++) r |= e2m1_away(v[i]) << (4 * i);
    return r;
}

// Two E2M1 codes (one byte) -> two fp32 values (exact), low nibble first.
FP4_DEV void e2m1x2_to_f32(uint32_t byte, float &lo, float &hi)
{
    uint32_t h2;
    asm("{\n\t.reg .b8 b;\n\t"
        "cvt.u8.u32 b, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b;\n\t}"
        : "=r"(h2)
        : "r"(byte));
    lo = __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFF)));
    hi = __half2float(__ushort_as_half((unsigned short)(h2 >> 16)));
}

// ---- E4M3 (unsigned use: NVFP4 block scale) ---------------------------------
FP4_DEV uint32_t e4m3_rn(float t)
{
    unsigned short h;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(0.0f), "f"(t));
    return h & 0xFFu;
}

FP4_DEV float e4m3_to_f32(uint32_t byte)
{
    uint32_t h2;
    unsigned short in = (unsigned short)(byte & 0xFF);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFF)));
}

// ---- E8M0 -----------------------------------------------------------------
// 2^e as an fp32 bit pattern for e in [-127, 127] (2^-127 is subnormal).
FP4_DEV float exp2i(int e)
{
    return (e >= -126) ? __uint_as_float((uint32_t)(e + 127) << 23) : __uint_as_float(0x00400000u);
}

// E8M0 scale byte -> 2^(byte - 127); 0xFF is NaN.
FP4_DEV float e8m0_to_f32(uint32_t byte) { return (byte == 0xFF) ? __uint_as_float(0x7FC00000u) : exp2i((int)byte - 127); }

// MXFP4 shared exponent from the block max (exact, from the exponent and
// mantissa bits).  amax = m * 2^E with m in [1, 2):
//   ceil rule : smallest e with amax <= 6 * 2^e  ->  E - 2 + (m > 1.5)
//   floor rule: floor(log2 amax) - 2             ->  E - 2
// amax == 0 gives -127; the result is clamped to [-127, 127].
FP4_DEV int mx_exponent(float amax, int floor_rule)
{
    uint32_t u = __float_as_uint(amax);
    if (u == 0) return -127;
    int E;
    uint32_t man;
    uint32_t ef = u >> 23;
    if (ef == 0) {  // subnormal: renormalise
        man = u & 0x7FFFFFu;
        int sh = __clz(man) - 8;
        man = (man << sh) & 0x7FFFFFu;
        E = -126 - sh;
    } else {
        man = u & 0x7FFFFFu;
        E = (int)ef - 127;
    }
    int e = E - 2 + ((!floor_rule && man > 0x400000u) ? 1 : 0);
    return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// ---- tile layout of the scale tensor ----------------------------------------
// Byte offset of logical scale (r, kb) in the 128x4 atom layout read by the
// block-scaled tcgen05 MMA (nkb4 = number of 4-scale column groups).
FP4_DEV int64_t scale_offset(int64_t r, int64_t kb, int64_t nkb4)
{
    return ((r >> 7) * nkb4 + (kb >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (kb & 3);
}

}  // namespace fp4
