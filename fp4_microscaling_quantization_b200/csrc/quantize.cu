// quantize.cu — HBM-streaming quantize / dequantize kernels for MXFP4 and
// NVFP4, with the optional block-diagonal Hadamard rotation fused in.
//
// Method: "Portable FP4 quantization (TransFP4)" §1.1 Eq.(1)
//   x^_i = s_g * s_b * Q_f(x_i / (s_g * s_b)),
// absmax block scales and nearest rounding (§3.1); the NVFP4 two-level scale
// ("4.5 FP8 and NVFP4/MXFP4" §4.1); the rotation H_k, k in {16,32,64,128},
// computed online for activations ("FP4 quantization analysis: MXFP4 vs
// NVFP4" §3.2.3, §3.3 fused online-rotation kernel).
//
// Work decomposition: one thread owns one 32-element unit of a row (one
// MXFP4 block or two NVFP4 blocks): four 16-byte loads, the block max in
// registers, one 16-byte store of 32 nibbles.  A Hadamard chunk of k <= 32
// lies inside one thread; k = 64 / 128 spans 2 / 4 neighbouring lanes and
// the last butterfly stages exchange values with shuffles.  Warps walk the
// tensor in a grid-stride loop of 32 consecutive units, so neighbouring
// lanes read and write neighbouring memory.
//
// Variants of the same loop: the MSE block-scale search (quantize_mse_kernel,
// §3.2.1 and §3.3 of the same page), the sparse residual lane
// (quantize_res_kernel, TransFP4 §2.3 Eq.(3)), the decode activation
// quantizer (act_quant_kernel, one cluster), and the offline helpers: the
// NVFP4 tensor-scale refinement and the MXFP4 -> NVFP4 scale binding.
#include <algorithm>
#include <map>
#include <mutex>

#include "encode.cuh"
#include "sm100.cuh"

namespace fp4 {

struct QuantArgs {
    const uint16_t *x;
    int64_t ld;             // row stride of x, elements
    int64_t units_per_row;  // cols / 32
    int64_t total_units;    // rows * units_per_row (< 2^32, checked by the launcher)
    FastDiv upr_div;        // division by units_per_row
    int64_t nkb4;           // ceil(blocks per row / 4)
    int64_t q_row_bytes;    // cols / 2
    uint8_t *q;
    uint8_t *s;
    float *gscale;
    float ck;               // RN(1/sqrt(k)) of the rotation
    int round_away;         // E2M1 ties to the larger magnitude
    int mx_floor;           // MX scale: floor rule
    int gscale_computed;    // NVFP4: *gscale was set by the amax pass (see amax_kernel)
    uint32_t *res;          // sparse residual lane (one word per unit), or null
    int wide;               // x and its row stride are 32-byte aligned: 32-byte loads
};

// Units processed per thread and loop trip: their loads are all issued
// before any is consumed, so each thread keeps UNITS x 64 bytes in flight.
constexpr int QUNITS = 2;  // quantize / amax
constexpr int DUNITS = 2;  // dequantize (16 bytes of nibbles per unit)

// Row and position in the row of unit u.
FP4_DEV void unit_rc(int64_t u, const FastDiv &upr, uint32_t &row, uint32_t &j)
{
    row = fastdiv((uint32_t)u, upr);
    j = (uint32_t)u - row * upr.d;
}

// Raw bytes of unit j of row `row` (4 x 16-byte loads, read-only path).
// 32-byte loads (one full sector per lane) when every unit starts on a
// 32-byte boundary (x and its row stride 32-byte aligned), else 16-byte ones.
FP4_DEV void ld_nc_v8(const void *p, uint4 &a, uint4 &b)
{
    asm volatile("ld.global.nc.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
                 : "l"(p));
}

FP4_DEV void ld_nc_v8_hint(const void *p, uint4 &a, uint4 &b, uint64_t pol)
{
    asm volatile("ld.global.nc.L2::cache_hint.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8], %9;"
                 : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
                 : "l"(p), "l"(pol));
}

FP4_DEV void fetch_unit(const uint16_t *x, int64_t ld, uint32_t row, uint32_t j, uint4 *w, bool wide = false)
{
    const uint4 *p = reinterpret_cast<const uint4 *>(x + (int64_t)row * ld + (int64_t)j * 32);
    if (wide) {
        ld_nc_v8(p, w[0], w[1]);
        ld_nc_v8(p + 2, w[2], w[3]);
        return;
    }
#pragma unroll
    for (int c = 0; c < 4; c++) w[c] = __ldg(p + c);
}

// L2 eviction policies for the two passes of an NVFP4 quantization with a
// computed tensor scale: the tensor-max pass marks x evict-last so that the
// encode pass, which marks it evict-first, finds it in L2 when it fits.
FP4_DEV uint64_t l2_policy_evict_last()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

FP4_DEV uint64_t l2_policy_evict_first()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

FP4_DEV void fetch_unit_hint(const uint16_t *x, int64_t ld, uint32_t row, uint32_t j, uint4 *w, uint64_t pol,
                             bool wide = false)
{
    const uint4 *p = reinterpret_cast<const uint4 *>(x + (int64_t)row * ld + (int64_t)j * 32);
    if (wide) {
        ld_nc_v8_hint(p, w[0], w[1], pol);
        ld_nc_v8_hint(p + 2, w[2], w[3], pol);
        return;
    }
#pragma unroll
    for (int c = 0; c < 4; c++)
        asm volatile("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                     : "=r"(w[c].x), "=r"(w[c].y), "=r"(w[c].z), "=r"(w[c].w)
                     : "l"(p + c), "l"(pol));
}

// s_g as left in *g by amax_kernel: max over CTAs of RN(amax_cta / 2688)
// equals RN(amax / 2688) (division by a positive constant and rounding are
// both monotonic), so only the all-zero and the non-finite cases remain,
// both mapped to 1.  The quantize kernel writes that 1 back; other CTAs may
// read 0 / inf or 1 meanwhile and decode either to the same s_g.
FP4_DEV float computed_global_scale(float v) { return (v > 0.0f && v <= kFltMax) ? v : 1.0f; }

FP4_DEV float read_global_scale(float *g, int computed)
{
    const float v = __ldcg(g);
    if (!computed) return v;
    const float sg = computed_global_scale(v);
    if (!(sg == v) && blockIdx.x == 0 && threadIdx.x == 0) atomicExch(g, sg);
    return sg;
}

// Encodes one rotated 32-element unit u (encode_unit, or encode_unit_mse for
// the MSE scale method) and stores its nibbles and scale byte(s) in the tile
// layout.
template <int FMT, bool MSE = false>
FP4_DEV void encode_store_unit(float *v, int64_t u, uint32_t row, uint32_t j, const QuantArgs &a, float sg, float six_sg,
                               const NvScaleTables *tab = nullptr)
{
    uint4 out;
    const uint32_t sb = MSE ? encode_unit_mse<FMT>(v, six_sg, a.round_away, tab, out)
                            : encode_unit<FMT>(v, sg, six_sg, a.round_away, a.mx_floor, out, tab);
    if (FMT == FP4_MXFP4)
        a.s[scale_offset(row, j, a.nkb4)] = (uint8_t)sb;
    else
        *reinterpret_cast<uint16_t *>(a.s + scale_offset(row, 2 * j, a.nkb4)) = (uint16_t)sb;
    *reinterpret_cast<uint4 *>(a.q + u * 16) = out;  // q rows are contiguous: row * cols/2 + j * 16 = u * 16
}

// ---------------------------------------------------------------------------
// NVFP4 tensor scale: every CTA folds RN(max |H_k x| over its part / 2688)
// into *gscale with an integer atomicMax (the bits of a non-negative float
// order like the float; *gscale must be 0 on entry).  The result is s_g =
// RN(amax / (6 * 448)) itself, or 0 for an all-zero tensor.
template <int HK, bool RES>
__global__ void __launch_bounds__(256) amax_kernel(QuantArgs a)
{
    grid_dep_launch();
    grid_dep_wait();
    const uint64_t pol = l2_policy_evict_last();
    const int lane = threadIdx.x & 31;
    const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    float m = 0.0f;
    for (int64_t base = warp * 32 * QUNITS; base < a.total_units; base += nwarps * 32 * QUNITS) {
        uint4 raw[QUNITS][4];
        uint32_t row[QUNITS] = {}, col[QUNITS] = {};
#pragma unroll
        for (int i = 0; i < QUNITS; i++) {
            const int64_t u = base + i * 32 + lane;
            if (u < a.total_units) {
                unit_rc(u, a.upr_div, row[i], col[i]);
                fetch_unit_hint(a.x, a.ld, row[i], col[i], raw[i], pol, a.wide);
            } else {
#pragma unroll
                for (int c = 0; c < 4; c++) raw[i][c] = make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int i = 0; i < QUNITS; i++) {
            float v[32];
            unpack_unit(raw[i], v);
            if (HK) fwht_unit<HK>(v, a.ck, lane);
            if (RES) extract_residual(v);  // the tensor scale of the FP4 stream
            m = fmaxf(m, absmax_tree<32>(v));
        }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    __shared__ float red[8];
    if (lane == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float b = red[0];
        for (int w = 1; w < (int)(blockDim.x >> 5); w++) b = fmaxf(b, red[w]);
        // integer order of non-negative float bits is float order
        atomicMax(reinterpret_cast<unsigned int *>(a.gscale), __float_as_uint(__fdiv_rn(b, 2688.0f)));
    }
}

// Clears the amax accumulator (a kernel rather than a memset node, so the
// whole sequence stays on the compute engine).
__global__ void zero_word_kernel(float *g)
{
    grid_dep_launch();
    grid_dep_wait();
    *g = 0.0f;
}

// ---------------------------------------------------------------------------
template <int FMT, int HK, bool MSE, bool RES = false>
FP4_DEV void quantize_body(const QuantArgs &a)
{
    grid_dep_launch();
    grid_dep_wait();
    const int lane = threadIdx.x & 31;
    const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;

    float sg = 1.0f, six_sg = 6.0f;
    if (FMT == FP4_NVFP4) {
        sg = read_global_scale(a.gscale, a.gscale_computed);
        six_sg = __fmul_rn(6.0f, sg);
    }
    const bool hinted = FMT == FP4_NVFP4 && a.gscale_computed;  // second read of x
    const uint64_t pol = l2_policy_evict_first();
    __shared__ NvScaleTables tab;  // NVFP4 only
    if (FMT == FP4_NVFP4) {
        nv_tables_fill(tab, sg, threadIdx.x, blockDim.x);
        __syncthreads();
    }

    // The MSE search is arithmetic-bound: one unit per trip keeps its
    // registers within three CTAs per SM.
    constexpr int NU = MSE ? 1 : QUNITS;
    for (int64_t base = warp * 32 * NU; base < a.total_units; base += nwarps * 32 * NU) {
        uint4 raw[NU][4];
        uint32_t row[NU] = {}, col[NU] = {};
#pragma unroll
        for (int i = 0; i < NU; i++) {
            const int64_t u = base + i * 32 + lane;
            if (u < a.total_units) {
                unit_rc(u, a.upr_div, row[i], col[i]);
                if (hinted) fetch_unit_hint(a.x, a.ld, row[i], col[i], raw[i], pol, a.wide); else fetch_unit(a.x, a.ld, row[i], col[i], raw[i], a.wide);
            } else {
#pragma unroll
                for (int c = 0; c < 4; c++) raw[i][c] = make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int i = 0; i < NU; i++) {
            const int64_t u = base + i * 32 + lane;
            const bool live = u < a.total_units;
            float v[32];
            unpack_unit(raw[i], v);
            if (HK) fwht_unit<HK>(v, a.ck, lane);
            if (!live) continue;
            if (RES) a.res[u] = extract_residual(v);

            encode_store_unit<FMT, MSE>(v, u, row[i], col[i], a, sg, six_sg, FMT == FP4_NVFP4 ? &tab : nullptr);
        }
    }
}

template <int FMT, int HK>
__global__ void __launch_bounds__(256) quantize_kernel(QuantArgs a)
{
    quantize_body<FMT, HK, false>(a);
}

// With the sparse residual lane.
template <int FMT, int HK>
__global__ void __launch_bounds__(256) quantize_res_kernel(QuantArgs a)
{
    quantize_body<FMT, HK, false, true>(a);
}

// The MSE scale search: arithmetic-bound, so sized for three CTAs per SM.
template <int FMT, int HK>
__global__ void __launch_bounds__(256, 3) quantize_mse_kernel(QuantArgs a)
{
    quantize_body<FMT, HK, true>(a);
}


// ---------------------------------------------------------------------------
// Activation quantization for the decode product (a few rows): one cluster of
// up to ACT_CTAS CTAs quantizes the whole tensor in a single launch.  Each
// thread owns the units u = (warp + i * warps) * 32 + lane, i < ACT_UPT, and
// when they cover the tensor it keeps their raw bytes in registers, so the
// NVFP4 tensor-max pass and the encode pass read x once.  The CTAs exchange
// their partial maxima through distributed shared memory: no global scratch,
// memset or second kernel.  The kernel also zeroes `nzero` words at `zero`
// (the split-K kernel's per-tile arrival counters) and the padding scale
// columns of the tensor's rows (with K not a multiple of 128 (MX) or 64
// (NV) the GEMM's last K step multiplies the zeros past K by them, so they
// must be finite), but not the padding rows, whose products the GEMM never
// stores.
constexpr int ACT_CTAS = 16, ACT_CTAS_PORTABLE = 8, ACT_THREADS = 256, ACT_UPT = 2;

// Loads units base + 32 i + lane (i < N) of the tensor, zeros past the end.
template <int N>
FP4_DEV void fetch_units(const QuantArgs &a, int64_t base, int64_t stride, int lane, uint4 (*raw)[4], uint32_t *row,
                         uint32_t *col)
{
#pragma unroll
    for (int i = 0; i < N; i++) {
        const int64_t u = base + i * stride + lane;
        row[i] = col[i] = 0;
        if (u < a.total_units) {
            unit_rc(u, a.upr_div, row[i], col[i]);
            fetch_unit(a.x, a.ld, row[i], col[i], raw[i]);
        } else {
#pragma unroll
            for (int c = 0; c < 4; c++) raw[i][c] = make_uint4(0, 0, 0, 0);
        }
    }
}

template <int FMT, int HK>
__global__ void __launch_bounds__(ACT_THREADS) act_quant_kernel(QuantArgs a, unsigned *zero, int nzero, int early)
{
    // Launched programmatically after the previous work in the stream.  The
    // dependent split-K kernel streams W before it waits, so by default it may
    // only start once everything before this kernel has finished: trigger
    // after the wait.  With `early` (the caller's weights are written by no
    // kernel that can still be running) it starts at once and streams W while
    // the previous work, and this kernel, finish.
    if (early) grid_dep_launch();
    grid_dep_wait();
    if (!early) grid_dep_launch();
    __shared__ float red[ACT_THREADS / 32];
    __shared__ float cta_max;
    const int lane = threadIdx.x & 31;
    const int64_t warp = (blockIdx.x * (int64_t)ACT_THREADS + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * ACT_THREADS) >> 5;
    for (int i = blockIdx.x * ACT_THREADS + threadIdx.x; i < nzero; i += gridDim.x * ACT_THREADS) zero[i] = 0u;
    {
        const int64_t nkb = a.units_per_row * (FMT == FP4_MXFP4 ? 1 : 2);
        const int pad = (int)(a.nkb4 * 4 - nkb);  // 0 .. 3
        const int64_t rows = a.units_per_row > 0 ? a.total_units / a.units_per_row : 0;
        for (int64_t i = blockIdx.x * ACT_THREADS + threadIdx.x; i < rows * pad; i += gridDim.x * ACT_THREADS)
            a.s[scale_offset(i / pad, nkb + i % pad, a.nkb4)] = 0;
    }

    const int64_t stride = nwarps * 32;  // units between a thread's consecutive units
    const bool cached = a.total_units <= stride * ACT_UPT;
    uint4 raw[ACT_UPT][4];
    uint32_t row[ACT_UPT], col[ACT_UPT];
    if (cached) fetch_units<ACT_UPT>(a, warp * 32, stride, lane, raw, row, col);

    float sg = 1.0f;
    if (FMT == FP4_NVFP4) {
        if (a.gscale_computed) {
            float m = 0.0f;
            if (cached) {
#pragma unroll
                for (int i = 0; i < ACT_UPT; i++) {
                    float v[32];
                    unpack_unit(raw[i], v);
                    if (HK) fwht_unit<HK>(v, a.ck, lane);
                    m = fmaxf(m, absmax_tree<32>(v));
                }
            } else {
                for (int64_t base = warp * 32; base < a.total_units; base += stride * QUNITS) {
                    uint4 r2[QUNITS][4];
                    uint32_t rw[QUNITS], cl[QUNITS];
                    fetch_units<QUNITS>(a, base, stride, lane, r2, rw, cl);
#pragma unroll
                    for (int i = 0; i < QUNITS; i++) {
                        float v[32];
                        unpack_unit(r2[i], v);
                        if (HK) fwht_unit<HK>(v, a.ck, lane);
                        m = fmaxf(m, absmax_tree<32>(v));
                    }
                }
            }
#pragma unroll
            for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
            if (lane == 0) red[threadIdx.x >> 5] = m;
            __syncthreads();
            if (threadIdx.x == 0) {
                float b = red[0];
                for (int w = 1; w < ACT_THREADS / 32; w++) b = fmaxf(b, red[w]);
                cta_max = b;
            }
            cluster_sync();  // every CTA's partial maximum is in place
            float t = 0.0f;
            for (unsigned r = 0; r < gridDim.x; r++) t = fmaxf(t, ld_shared_cluster_f32(mapa_shared(smem_u32(&cta_max), r)));
            cluster_sync();  // no CTA leaves while another still reads its shared memory
            sg = nv_global_from_amax(t);
            if (blockIdx.x == 0 && threadIdx.x == 0) *a.gscale = sg;
        } else {
            sg = *a.gscale;
        }
    }
    const float six_sg = __fmul_rn(6.0f, sg);

    if (cached) {
#pragma unroll
        for (int i = 0; i < ACT_UPT; i++) {
            const int64_t u = warp * 32 + i * stride + lane;
            float v[32];
            unpack_unit(raw[i], v);
            if (HK) fwht_unit<HK>(v, a.ck, lane);
            if (u < a.total_units) encode_store_unit<FMT>(v, u, row[i], col[i], a, sg, six_sg);
        }
        return;
    }
    for (int64_t base = warp * 32; base < a.total_units; base += stride * QUNITS) {
        uint4 r2[QUNITS][4];
        uint32_t rw[QUNITS], cl[QUNITS];
        fetch_units<QUNITS>(a, base, stride, lane, r2, rw, cl);
#pragma unroll
        for (int i = 0; i < QUNITS; i++) {
            const int64_t u = base + i * stride + lane;
            float v[32];
            unpack_unit(r2[i], v);
            if (HK) fwht_unit<HK>(v, a.ck, lane);
            if (u < a.total_units) encode_store_unit<FMT>(v, u, rw[i], cl[i], a, sg, six_sg);
        }
    }
}

// Zero the padding bytes of the scale tile layout: scale columns
// [nkb, 4*nkb4) of real rows, and every byte of rows [rows, pad128(rows)).
__global__ void scale_pad_kernel(uint8_t *s, int64_t rows, int64_t nkb, int64_t nkb4)
{
    grid_dep_launch();
    grid_dep_wait();
    const int64_t cpad = nkb4 * 4 - nkb;
    const int64_t rows_p = (rows + 127) / 128 * 128;
    const int64_t n1 = rows * cpad;
    const int64_t n2 = (rows_p - rows) * nkb4 * 4;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n1 + n2;
         i += (int64_t)gridDim.x * blockDim.x) {
        int64_t r, kb;
        if (i < n1) {
            r = i / cpad;
            kb = nkb + (i - r * cpad);
        } else {
            const int64_t t = i - n1;
            r = rows + t / (nkb4 * 4);
            kb = t % (nkb4 * 4);
        }
        s[scale_offset(r, kb, nkb4)] = 0;
    }
}

// ---------------------------------------------------------------------------
struct DequantArgs {
    const uint8_t *q;
    const uint8_t *s;
    const float *gscale;
    int64_t units_per_row;
    int64_t total_units;    // < 2^32, checked by the launcher
    FastDiv upr_div;        // division by units_per_row
    int64_t nkb4;
    int64_t q_row_bytes;
    int64_t cols;
    void *out;
    float ck;
    const uint32_t *res;    // sparse residual lane, or null
};

template <int FMT, int HK, int BF16OUT, bool RES = false>
__global__ void __launch_bounds__(256) dequantize_kernel(DequantArgs a)
{
    grid_dep_launch();
    grid_dep_wait();
    constexpr int NC = BF16OUT ? 4 : 8;  // 16-byte output chunks per 32-element unit
    __shared__ uint4 stage_all[8 * 32 * NC];
    const int lane = threadIdx.x & 31;
    const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const float sg = (FMT == FP4_NVFP4) ? *a.gscale : 1.0f;

    for (int64_t base = warp * 32 * DUNITS; base < a.total_units; base += nwarps * 32 * DUNITS) {
        uint4 raw[DUNITS];
        uint32_t sraw[DUNITS], rres[DUNITS];
#pragma unroll
        for (int i = 0; i < DUNITS; i++) {
            const int64_t u = base + i * 32 + lane;
            raw[i] = make_uint4(0, 0, 0, 0);
            sraw[i] = 0;
            rres[i] = 0;
            if (u < a.total_units) {
                if (RES) rres[i] = __ldg(a.res + u);
                uint32_t row, j;
                unit_rc(u, a.upr_div, row, j);
                raw[i] = __ldg(reinterpret_cast<const uint4 *>(a.q + u * 16));
                sraw[i] = (FMT == FP4_MXFP4)
                              ? (uint32_t)__ldg(a.s + scale_offset(row, j, a.nkb4))
                              : (uint32_t)__ldg(reinterpret_cast<const unsigned short *>(a.s + scale_offset(row, 2 * j, a.nkb4)));
            }
        }
#pragma unroll
        for (int i = 0; i < DUNITS; i++) {
            const int64_t u = base + i * 32 + lane;
            const bool live = u < a.total_units;
            float v[32];
            if (live) {
                const uint4 w = raw[i];
                const uint32_t words[4] = {w.x, w.y, w.z, w.w};
                float d0, d1;
                if (FMT == FP4_MXFP4) {
                    d0 = d1 = e8m0_to_f32(sraw[i]);
                } else if (FMT == FP4_MXFP4_16) {
                    d0 = e8m0_to_f32(sraw[i] & 0xFF);
                    d1 = e8m0_to_f32(sraw[i] >> 8);
                } else {
                    const uint32_t sb2 = sraw[i];
                    d0 = __fmul_rn(sg, e4m3_to_f32(sb2 & 0xFF));
                    d1 = __fmul_rn(sg, e4m3_to_f32(sb2 >> 8));
                }
#pragma unroll
                for (int c = 0; c < 4; c++) {
#pragma unroll
                    for (int b = 0; b < 4; b++) {
                        float lo, hi;
                        e2m1x2_to_f32((words[c] >> (8 * b)) & 0xFF, lo, hi);
                        const float d = (c < 2) ? d0 : d1;
                        v[8 * c + 2 * b] = __fmul_rn(d, lo);
                        v[8 * c + 2 * b + 1] = __fmul_rn(d, hi);
                    }
                }
                if (RES) {
                    // TransFP4 Eq.(3): the FP4 stream plus the residual lane
                    const int idx = (int)((rres[i] >> 16) & 31u);
                    const float r = __uint_as_float((rres[i] & 0xFFFFu) << 16);
#pragma unroll
                    for (int e = 0; e < 32; e++)
                        if (e == idx) v[e] = __fadd_rn(v[e], r);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; i++) v[i] = 0.0f;
            }
            if (HK) fwht_unit<HK>(v, a.ck, lane);

            // Stage the unit's output in shared memory (16-byte chunks, XOR
            // swizzled so both the row-wise writes and the chunk-wise reads are
            // free of bank conflicts), then store it as whole 512-byte warp
            // segments: the warp's 32 units are contiguous in the output.
            uint4 *stage = stage_all + (threadIdx.x >> 5) * (32 * NC);
            if (BF16OUT) {
#pragma unroll
                for (int c = 0; c < 4; c++) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        __nv_bfloat162 h = __floats2bfloat162_rn(v[8 * c + 2 * e], v[8 * c + 2 * e + 1]);
                        w[e] = *reinterpret_cast<uint32_t *>(&h);
                    }
                    stage[lane * NC + (c ^ ((lane >> 1) & 3))] = make_uint4(w[0], w[1], w[2], w[3]);
                }
            } else {
#pragma unroll
                for (int c = 0; c < 8; c++)
                    stage[lane * NC + (c ^ (lane & 7))] =
                        make_uint4(__float_as_uint(v[4 * c]), __float_as_uint(v[4 * c + 1]),
                                   __float_as_uint(v[4 * c + 2]), __float_as_uint(v[4 * c + 3]));
            }
            __syncwarp();
            const int64_t ubase = base + i * 32;
            uint4 *out16 = reinterpret_cast<uint4 *>(a.out) + ubase * NC;
#pragma unroll
            for (int k = 0; k < NC; k++) {
                const int ch = k * 32 + lane;   // chunk within the warp's segment
                const int un = ch / NC, c = ch % NC;
                const int cp = BF16OUT ? (c ^ ((un >> 1) & 3)) : (c ^ (un & 7));
                if (ubase + un < a.total_units) out16[ch] = stage[un * NC + cp];
            }
            __syncwarp();
        }
    }
}

// ---------------------------------------------------------------------------
// Host launchers (called from capi.cu after validation).
static int grid_for(int64_t total_units, int sms, int units_per_thread)
{
    const int64_t warps = (total_units + 32 * units_per_thread - 1) / (32 * units_per_thread);
    const int64_t blocks = (warps + 7) / 8;  // 8 warps per 256-thread block
    const int64_t cap = (int64_t)sms * 8;
    return (int)(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

template <int FMT, bool MSE>
static void (*quant_kernel_for(int hk))(QuantArgs)
{
    switch (hk) {
    case 0: return MSE ? quantize_mse_kernel<FMT, 0> : quantize_kernel<FMT, 0>;
    case 16: return MSE ? quantize_mse_kernel<FMT, 16> : quantize_kernel<FMT, 16>;
    case 32: return MSE ? quantize_mse_kernel<FMT, 32> : quantize_kernel<FMT, 32>;
    case 64: return MSE ? quantize_mse_kernel<FMT, 64> : quantize_kernel<FMT, 64>;
    case 128: return MSE ? quantize_mse_kernel<FMT, 128> : quantize_kernel<FMT, 128>;
    }
    return nullptr;
}

template <int FMT>
static void (*quant_res_kernel_for(int hk))(QuantArgs)
{
    switch (hk) {
    case 0: return quantize_res_kernel<FMT, 0>;
    case 16: return quantize_res_kernel<FMT, 16>;
    case 32: return quantize_res_kernel<FMT, 32>;
    case 64: return quantize_res_kernel<FMT, 64>;
    case 128: return quantize_res_kernel<FMT, 128>;
    }
    return nullptr;
}

template <int FMT>
static void (*quant_kernel_pick(int hk, int mse, bool res))(QuantArgs)
{
    return res ? quant_res_kernel_for<FMT>(hk) : mse ? quant_kernel_for<FMT, true>(hk) : quant_kernel_for<FMT, false>(hk);
}

template <bool RES>
static void (*amax_kernel_for(int hk))(QuantArgs)
{
    switch (hk) {
    case 0: return amax_kernel<0, RES>;
    case 16: return amax_kernel<16, RES>;
    case 32: return amax_kernel<32, RES>;
    case 64: return amax_kernel<64, RES>;
    case 128: return amax_kernel<128, RES>;
    }
    return nullptr;
}

// Quantize launch sequence (see the note on `pdl` below).
cudaError_t launch_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, int fmt,
                            int hk, float ck, int round_away, int mx_floor, int mse, int gscale_given,
                            uint8_t *q, uint8_t *s, float *gscale, int sms, cudaStream_t st, bool pdl, uint32_t *res)
{
    QuantArgs a;
    a.x = x;
    a.ld = ld;
    a.units_per_row = cols / 32;
    a.total_units = rows * (cols / 32);
    if (a.total_units >= (int64_t(1) << 32)) return cudaErrorInvalidValue;
    a.upr_div = make_fastdiv((uint32_t)(a.units_per_row > 0 ? a.units_per_row : 1));
    const int64_t nkb = cols / (fmt == FP4_MXFP4 ? 32 : 16);
    a.nkb4 = (nkb + 3) / 4;
    a.q_row_bytes = cols / 2;
    a.q = q;
    a.s = s;
    a.gscale = gscale;
    a.ck = ck;
    a.round_away = round_away;
    a.mx_floor = mx_floor;
    a.gscale_computed = (fmt == FP4_NVFP4 && !gscale_given) ? 1 : 0;
    a.res = res;
    a.wide = ((reinterpret_cast<uintptr_t>(x) & 31) == 0 && (ld * 2) % 32 == 0) ? 1 : 0;
    const int grid = grid_for(a.total_units, sms, QUNITS);
    void (*qk)(QuantArgs) = fmt == FP4_MXFP4   ? quant_kernel_pick<FP4_MXFP4>(hk, mse, res != nullptr)
                            : fmt == FP4_NVFP4 ? quant_kernel_pick<FP4_NVFP4>(hk, mse, res != nullptr)
                                               : quant_kernel_pick<FP4_MXFP4_16>(hk, mse, res != nullptr);
    void (*ak)(QuantArgs) = res ? amax_kernel_for<true>(hk) : amax_kernel_for<false>(hk);
    if (!qk || !ak) return cudaErrorInvalidValue;
    cudaError_t err = cudaSuccess;
    // With `pdl` every launch, the first included, may start while its
    // predecessor drains: each kernel waits for it before touching memory,
    // and none reads anything before that wait.
    if (a.gscale_computed) {
        if ((err = launch_k(zero_word_kernel, dim3(1), dim3(1), 0, st, pdl, gscale)) != cudaSuccess) return err;
        if ((err = launch_k(ak, dim3(grid), dim3(256), 0, st, pdl, a)) != cudaSuccess) return err;
    }
    if (a.total_units > 0 || a.gscale_computed) {  // an empty NVFP4 tensor still gets s_g = 1
        // NVFP4 (absmax scales, k <= 32): one resident wave (3 CTAs per SM at
        // its register count), so fewer CTAs build the scale tables; with the
        // rotation's cross-lane stages or the residual lane the longer grid
        // balances better
        const int qgrid = (fmt == FP4_NVFP4 && !mse && !res && hk <= 32 && grid > sms * 3) ? sms * 3 : grid;
        if ((err = launch_k(qk, dim3(qgrid), dim3(256), 0, st, pdl, a)) != cudaSuccess) return err;
    }
    const int64_t rows_p = (rows + 127) / 128 * 128;
    const int64_t npad = rows * (a.nkb4 * 4 - nkb) + (rows_p - rows) * a.nkb4 * 4;
    if (npad > 0) {
        int g = (int)((npad + 255) / 256);
        if (g > sms * 4) g = sms * 4;
        if ((err = launch_k(scale_pad_kernel, dim3(g), dim3(256), 0, st, pdl, s, rows, nkb, a.nkb4)) != cudaSuccess)
            return err;
    }
    return cudaSuccess;
}


template <int FMT>
static void (*act_kernel_for(int hk))(QuantArgs, unsigned *, int, int)
{
    switch (hk) {
    case 0: return act_quant_kernel<FMT, 0>;
    case 16: return act_quant_kernel<FMT, 16>;
    case 32: return act_quant_kernel<FMT, 32>;
    case 64: return act_quant_kernel<FMT, 64>;
    case 128: return act_quant_kernel<FMT, 128>;
    }
    return nullptr;
}

// Cluster size of the activation quantizer: ACT_CTAS (a non-portable size)
// where the device schedules such clusters, else the portable ACT_CTAS_PORTABLE.
// Decided once per kernel instance and device (the attribute it sets belongs
// to the current device's context).
static int act_cluster_size(void (*k)(QuantArgs, unsigned *, int, int))
{
    static std::mutex mu;
    static std::map<std::pair<const void *, int>, int> sizes;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return ACT_CTAS_PORTABLE;
    }
    const std::pair<const void *, int> key(reinterpret_cast<const void *>(k), dev);
    std::lock_guard<std::mutex> lock(mu);
    auto it = sizes.find(key);
    if (it != sizes.end()) return it->second;
    int n = ACT_CTAS_PORTABLE;
    bool refused = false;  // a refused call leaves its error for cudaGetLastError: clear only ours
    if (cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
        refused = true;
    } else {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(ACT_CTAS);
        cfg.blockDim = dim3(ACT_THREADS);
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = ACT_CTAS;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, k, &cfg) != cudaSuccess)
            refused = true;
        else if (clusters > 0)
            n = ACT_CTAS;
    }
    if (refused) cudaGetLastError();
    sizes[key] = n;
    return n;
}

// Single-launch quantization of a small activation tensor (see
// act_quant_kernel).  Only the NVFP4 tensor maximum needs the CTAs to form a
// cluster; without it the CTAs are scheduled one by one, which a device
// still busy with the previous kernel can do sooner.
cudaError_t launch_act_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, int fmt, int hk, float ck,
                                int round_away, int mx_floor, int gscale_given, uint8_t *q, uint8_t *s, float *gscale,
                                unsigned *zero, int nzero, int early, cudaStream_t st)
{
    QuantArgs a;
    a.x = x;
    a.ld = ld;
    a.units_per_row = cols / 32;
    a.total_units = rows * (cols / 32);
    if (a.total_units >= (int64_t(1) << 32)) return cudaErrorInvalidValue;
    a.upr_div = make_fastdiv((uint32_t)(a.units_per_row > 0 ? a.units_per_row : 1));
    const int64_t nkb = cols / (fmt == FP4_MXFP4 ? 32 : 16);
    a.nkb4 = (nkb + 3) / 4;
    a.q_row_bytes = cols / 2;
    a.q = q;
    a.s = s;
    a.gscale = gscale;
    a.ck = ck;
    a.round_away = round_away;
    a.mx_floor = mx_floor;
    a.gscale_computed = (fmt == FP4_NVFP4 && !gscale_given) ? 1 : 0;
    a.res = nullptr;
    a.wide = 0;
    void (*k)(QuantArgs, unsigned *, int, int) = fmt == FP4_MXFP4   ? act_kernel_for<FP4_MXFP4>(hk)
                                                 : fmt == FP4_NVFP4 ? act_kernel_for<FP4_NVFP4>(hk)
                                                                    : act_kernel_for<FP4_MXFP4_16>(hk);
    if (!k) return cudaErrorInvalidValue;
    const bool cluster = a.gscale_computed != 0;
    const int ctas = cluster ? act_cluster_size(k) : ACT_CTAS;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ctas);
    cfg.blockDim = dim3(ACT_THREADS);
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    // May start while the previous kernel drains (its launch latency is then
    // hidden); the kernel waits for it before touching memory.
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = ctas;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = cluster ? 2 : 1;
    count_launches(1);
    return cudaLaunchKernelEx(&cfg, k, a, zero, nzero, early);
}

template <int FMT, int BF, bool RES>
static void (*deq_kernel_for(int hk))(DequantArgs)
{
    switch (hk) {
    case 0: return dequantize_kernel<FMT, 0, BF, RES>;
    case 16: return dequantize_kernel<FMT, 16, BF, RES>;
    case 32: return dequantize_kernel<FMT, 32, BF, RES>;
    case 64: return dequantize_kernel<FMT, 64, BF, RES>;
    case 128: return dequantize_kernel<FMT, 128, BF, RES>;
    }
    return nullptr;
}

template <int FMT>
static void (*deq_kernel_pick(int hk, int bf16out, bool res))(DequantArgs)
{
    return res ? (bf16out ? deq_kernel_for<FMT, 1, true>(hk) : deq_kernel_for<FMT, 0, true>(hk))
               : (bf16out ? deq_kernel_for<FMT, 1, false>(hk) : deq_kernel_for<FMT, 0, false>(hk));
}

// ---------------------------------------------------------------------------
// Alternating refinement of the NVFP4 tensor scale ("FP4 quantization
// analysis: MXFP4 vs NVFP4" §3.2.1: group and global scales optimised in
// turn).  From the absmax s_g, each round quantizes with the MSE block-scale
// search under the current s_g, measures E = sum (x_i - y_i)^2 over the
// rotated values and their reconstructions, and moves s_g to the least-
// squares scale of the chosen codes, sum x_i u_i / sum u_i^2 with u_i =
// dec(s_b) dec(q_i); the s_g of the smallest E is kept.  All sums are fp64
// in a fixed order (a unit's 32 values, a row's units, the rows), so the
// result does not depend on the launch shape.
struct RefineState {
    double best_err;
    float cur_sg;   // the s_g the current round quantizes with
    float best_sg;
};

// Per unit: (sum x u, sum u u, sum e e) of the current round, in value order.
template <int HK>
__global__ void __launch_bounds__(256) nv_unit_stats_kernel(QuantArgs a, const RefineState *st, double *stats)
{
    grid_dep_launch();
    grid_dep_wait();
    const float sg = st->cur_sg;
    const int lane = threadIdx.x & 31;
    const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t base = warp * 32; base < a.total_units; base += nwarps * 32) {
        const int64_t u = base + lane;
        const bool live = u < a.total_units;
        uint4 raw[4];
        uint32_t row = 0, j = 0;
        if (live) {
            unit_rc(u, a.upr_div, row, j);
            fetch_unit(a.x, a.ld, row, j, raw);
        } else {
#pragma unroll
            for (int c = 0; c < 4; c++) raw[c] = make_uint4(0, 0, 0, 0);
        }
        float v[32];
        unpack_unit(raw, v);
        if (HK) fwht_unit<HK>(v, a.ck, lane);  // the whole warp takes part
        if (!live) continue;
        const uint4 qw = *reinterpret_cast<const uint4 *>(a.q + u * 16);
        const uint32_t sb2 = *reinterpret_cast<const uint16_t *>(a.s + scale_offset(row, 2 * j, a.nkb4));
        const uint32_t words[4] = {qw.x, qw.y, qw.z, qw.w};
        double sxu = 0.0, suu = 0.0, see = 0.0;
#pragma unroll
        for (int h = 0; h < 2; h++) {
            const float dsb = e4m3_to_f32((sb2 >> (8 * h)) & 0xFF);
            const float d = __fmul_rn(sg, dsb);
#pragma unroll
            for (int b = 0; b < 8; b++) {
                const int i0 = 16 * h + 2 * b;
                float q0, q1;
                e2m1x2_to_f32((words[i0 >> 3] >> (4 * (i0 & 7))) & 0xFF, q0, q1);
                const float qv[2] = {q0, q1};
#pragma unroll
                for (int e = 0; e < 2; e++) {
                    const double ui = __dmul_rn((double)dsb, (double)qv[e]);
                    const float yi = __fmul_rn(d, qv[e]);
                    const double xi = (double)v[i0 + e];
                    const double er = __dsub_rn(xi, (double)yi);
                    sxu = __dadd_rn(sxu, __dmul_rn(xi, ui));
                    suu = __dadd_rn(suu, __dmul_rn(ui, ui));
                    see = __dadd_rn(see, __dmul_rn(er, er));
                }
            }
        }
        stats[u * 3 + 0] = sxu;
        stats[u * 3 + 1] = suu;
        stats[u * 3 + 2] = see;
    }
}

// Per row: the row's unit sums in unit order.
__global__ void nv_row_stats_kernel(const double *stats, int64_t rows, int64_t upr, double *row_stats)
{
    grid_dep_launch();
    grid_dep_wait();
    for (int64_t r = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; r < rows; r += (int64_t)gridDim.x * blockDim.x) {
        double a0 = 0.0, a1 = 0.0, a2 = 0.0;
        for (int64_t u = 0; u < upr; u++) {
            const double *p = stats + (r * upr + u) * 3;
            a0 = __dadd_rn(a0, p[0]);
            a1 = __dadd_rn(a1, p[1]);
            a2 = __dadd_rn(a2, p[2]);
        }
        row_stats[r * 3 + 0] = a0;
        row_stats[r * 3 + 1] = a1;
        row_stats[r * 3 + 2] = a2;
    }
}

// One thread: the round's totals in row order, the best s_g so far (also
// written to `out`), and the next round's s_g.
__global__ void nv_refine_step_kernel(const double *row_stats, int64_t rows, int round, RefineState *st, float *out)
{
    grid_dep_launch();
    grid_dep_wait();
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    double sxu = 0.0, suu = 0.0, see = 0.0;
    for (int64_t r = 0; r < rows; r++) {
        sxu = __dadd_rn(sxu, row_stats[r * 3 + 0]);
        suu = __dadd_rn(suu, row_stats[r * 3 + 1]);
        see = __dadd_rn(see, row_stats[r * 3 + 2]);
    }
    if (round == 0 || see < st->best_err) {
        st->best_err = see;
        st->best_sg = st->cur_sg;
    }
    if (suu > 0.0) {
        const float nxt = __double2float_rn(__ddiv_rn(sxu, suu));
        if (nxt > 0.0f && nxt <= kFltMax) st->cur_sg = nxt;
    }
    *out = st->best_sg;
}

template <int HK>
static void (*unit_stats_kernel_for_k())(QuantArgs, const RefineState *, double *)
{
    return nv_unit_stats_kernel<HK>;
}

size_t nv_refine_workspace_bytes(int64_t rows, int64_t cols)
{
    const int64_t units = rows * (cols / 32);
    return 256 + (size_t)((units * 3 * 8 + 255) / 256 * 256) + (size_t)((rows * 3 * 8 + 255) / 256 * 256);
}

cudaError_t launch_nv_refine(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, int hk, float ck,
                             int round_away, int rounds, uint8_t *q, uint8_t *s, void *ws, float *gscale, int sms,
                             cudaStream_t st)
{
    uint8_t *base = static_cast<uint8_t *>(ws);
    RefineState *state = reinterpret_cast<RefineState *>(base);
    const int64_t units = rows * (cols / 32);
    double *ustats = reinterpret_cast<double *>(base + 256);
    double *rstats = reinterpret_cast<double *>(base + 256 + (units * 3 * 8 + 255) / 256 * 256);
    // the absmax s_g, computed into state->cur_sg
    cudaError_t e = launch_quantize(x, rows, cols, ld, FP4_NVFP4, hk, ck, round_away, 0, 0, 0, q, s, &state->cur_sg,
                                    sms, st, true, nullptr);
    if (e != cudaSuccess) return e;
    QuantArgs a;
    a.x = x;
    a.ld = ld;
    a.units_per_row = cols / 32;
    a.total_units = units;
    a.upr_div = make_fastdiv((uint32_t)(a.units_per_row > 0 ? a.units_per_row : 1));
    a.nkb4 = (cols / 16 + 3) / 4;
    a.q_row_bytes = cols / 2;
    a.q = q;
    a.s = s;
    a.gscale = &state->cur_sg;
    a.ck = ck;
    a.round_away = round_away;
    a.mx_floor = 0;
    a.gscale_computed = 0;
    a.res = nullptr;
    a.wide = 0;
    void (*uk)(QuantArgs, const RefineState *, double *) = nullptr;
    switch (hk) {
    case 0: uk = unit_stats_kernel_for_k<0>(); break;
    case 16: uk = unit_stats_kernel_for_k<16>(); break;
    case 32: uk = unit_stats_kernel_for_k<32>(); break;
    case 64: uk = unit_stats_kernel_for_k<64>(); break;
    case 128: uk = unit_stats_kernel_for_k<128>(); break;
    }
    if (!uk) return cudaErrorInvalidValue;
    const int g_units = grid_for(units, sms, 1);
    const int g_rows = (int)std::min<int64_t>((rows + 127) / 128, (int64_t)sms * 4);
    for (int r = 0; r < rounds; r++) {
        if ((e = launch_quantize(x, rows, cols, ld, FP4_NVFP4, hk, ck, round_away, 0, 1, 1, q, s, &state->cur_sg, sms,
                                 st, true, nullptr)) != cudaSuccess)
            return e;
        if ((e = launch_k(uk, dim3(g_units), dim3(256), 0, st, true, a, (const RefineState *)state, ustats)) !=
            cudaSuccess)
            return e;
        if ((e = launch_k(nv_row_stats_kernel, dim3(g_rows > 0 ? g_rows : 1), dim3(128), 0, st, true,
                          (const double *)ustats, rows, (int64_t)(cols / 32), rstats)) != cudaSuccess)
            return e;
        if ((e = launch_k(nv_refine_step_kernel, dim3(1), dim3(32), 0, st, true, (const double *)rstats, rows, r,
                          state, gscale)) != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

// ---------------------------------------------------------------------------
// MXFP4 -> NVFP4 scale repacking ("Portable FP4 quantization (TransFP4)"
// §2.5, §3.4: an artifact is bound late to the backend's native format).  The
// E2M1 elements stay; each 32-block scale 2^e becomes two 16-block E4M3
// scales 2^(e - E) under s_g = 2^E, E = max(e_max - 8, -126), so that
// s_g * s_b = 2^e: the largest block scale lands on 2^8, the largest power of
// two E4M3 holds.  Blocks more than 17 binades below it take the E4M3
// rounding of 2^(e - E) (0 from 2^-10 down).  E8M0 NaN becomes E4M3 NaN.

// Position (row, scale column) of byte i of a scale tile layout with nkb4
// 4-column groups (the inverse of scale_offset).
FP4_DEV void scale_position(int64_t i, int64_t nkb4, int64_t &r, int64_t &kb)
{
    const int64_t atom = i >> 9, o = i & 511;
    r = (atom / nkb4) * 128 + ((o & 15) >> 2) * 32 + (o >> 4);
    kb = (atom % nkb4) * 4 + (o & 3);
}

__global__ void set_word_kernel(float *g, float v)
{
    grid_dep_launch();
    grid_dep_wait();
    *g = v;
}

// *g = max(*g, 2^(e_max - 8)) over the real MXFP4 scale bytes, as an integer
// max of the float bits (positive floats order like their bits).  2^(b - 135)
// has the bits (b - 8) << 23 for a byte b >= 9; smaller bytes fall under the
// 2^-126 that *g starts from.
__global__ void mx_scale_max_kernel(const uint8_t *s, int64_t rows, int64_t nkb, int64_t nkb4, float *g)
{
    grid_dep_launch();
    grid_dep_wait();
    uint32_t best = 0;
    const int64_t n = (rows + 127) / 128 * 128 * nkb4 * 4;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        int64_t r, kb;
        scale_position(i, nkb4, r, kb);
        const uint32_t b = s[i];
        if (r < rows && kb < nkb && b != 0xFFu && b >= 9u) best = max(best, (b - 8u) << 23);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) best = max(best, __shfl_xor_sync(0xFFFFFFFFu, best, o));
    if ((threadIdx.x & 31) == 0 && best) atomicMax(reinterpret_cast<unsigned int *>(g), best);
}

// Writes every byte of the NVFP4 scale layout: the repacked scale of real
// positions, 0 in the padding.
__global__ void mx_to_nv_scale_kernel(const uint8_t *s_mx, int64_t rows, int64_t nkb, int64_t nkb4_mx, int64_t nkb4_nv,
                                      const float *g, uint8_t *s_nv)
{
    grid_dep_launch();
    grid_dep_wait();
    const int E = (int)((__float_as_uint(*g) >> 23) & 0xFF) - 127;
    const int64_t n = (rows + 127) / 128 * 128 * nkb4_nv * 4;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        int64_t r, kb16;
        scale_position(i, nkb4_nv, r, kb16);
        uint32_t v = 0;
        if (r < rows && kb16 < 2 * nkb) {
            const uint32_t b = s_mx[scale_offset(r, kb16 >> 1, nkb4_mx)];
            if (b == 0xFFu) {
                v = 0x7Fu;
            } else {
                const int d = (int)b - 127 - E;
                v = e4m3_rn(exp2i(d < -127 ? -127 : d));
            }
        }
        s_nv[i] = (uint8_t)v;
    }
}

cudaError_t launch_mx_to_nv_scales(const uint8_t *s_mx, int64_t rows, int64_t cols, uint8_t *s_nv, float *gscale,
                                   int sms, cudaStream_t st)
{
    const int64_t nkb = cols / 32, nkb4_mx = (nkb + 3) / 4, nkb4_nv = (2 * nkb + 3) / 4;
    cudaError_t e = launch_k(set_word_kernel, dim3(1), dim3(1), 0, st, true, gscale, 1.17549435082228750797e-38f);
    if (e != cudaSuccess || rows == 0 || nkb == 0) return e;
    const int64_t n_mx = (rows + 127) / 128 * 128 * nkb4_mx * 4, n_nv = (rows + 127) / 128 * 128 * nkb4_nv * 4;
    const int g1 = (int)std::min<int64_t>((n_mx + 255) / 256, (int64_t)sms * 4);
    const int g2 = (int)std::min<int64_t>((n_nv + 255) / 256, (int64_t)sms * 4);
    if ((e = launch_k(mx_scale_max_kernel, dim3(g1), dim3(256), 0, st, true, s_mx, rows, nkb, nkb4_mx, gscale)) !=
        cudaSuccess)
        return e;
    return launch_k(mx_to_nv_scale_kernel, dim3(g2), dim3(256), 0, st, true, s_mx, rows, nkb, nkb4_mx, nkb4_nv,
                    (const float *)gscale, s_nv);
}

cudaError_t launch_dequantize(const uint8_t *q, const uint8_t *s, const float *gscale, int64_t rows,
                              int64_t cols, int fmt, int hk, float ck, int bf16out, void *out,
                              int sms, cudaStream_t st, const uint32_t *res)
{
    DequantArgs a;
    a.q = q;
    a.s = s;
    a.gscale = gscale;
    a.units_per_row = cols / 32;
    a.total_units = rows * (cols / 32);
    if (a.total_units >= (int64_t(1) << 32)) return cudaErrorInvalidValue;
    a.upr_div = make_fastdiv((uint32_t)(a.units_per_row > 0 ? a.units_per_row : 1));
    const int64_t nkb = cols / (fmt == FP4_MXFP4 ? 32 : 16);
    a.nkb4 = (nkb + 3) / 4;
    a.q_row_bytes = cols / 2;
    a.cols = cols;
    a.out = out;
    a.ck = ck;
    a.res = res;
    if (a.total_units == 0) return cudaSuccess;
    const int grid = grid_for(a.total_units, sms, DUNITS);
    void (*k)(DequantArgs) = fmt == FP4_MXFP4   ? deq_kernel_pick<FP4_MXFP4>(hk, bf16out, res != nullptr)
                             : fmt == FP4_NVFP4 ? deq_kernel_pick<FP4_NVFP4>(hk, bf16out, res != nullptr)
                                                : deq_kernel_pick<FP4_MXFP4_16>(hk, bf16out, res != nullptr);
    if (!k) return cudaErrorInvalidValue;
    // programmatic launch: the kernel waits for its predecessor before touching memory
    return launch_k(k, dim3(grid), dim3(256), 0, st, true, a);
}

}  // namespace fp4
