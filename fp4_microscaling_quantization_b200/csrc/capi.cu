// capi.cu — the extern "C" boundary declared in include/fp4.h: host-side
// validation of every argument, then stream-ordered launches.  No entry point
// allocates or frees device memory or synchronizes the host (except
// fp4_check_device_status, which is documented to).
#include <math.h>

#include <atomic>

#include "common.cuh"

namespace fp4 {
cudaError_t launch_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, int fmt,
                            int hk, float ck, int round_away, int mx_floor, int mse, int gscale_given,
                            uint8_t *q, uint8_t *s, float *gscale, int sms, cudaStream_t st, bool pdl,
                            uint32_t *res);
cudaError_t launch_dequantize(const uint8_t *q, const uint8_t *s, const float *gscale, int64_t rows,
                              int64_t cols, int fmt, int hk, float ck, int bf16out, void *out,
                              int sms, cudaStream_t st, const uint32_t *res);
cudaError_t launch_gemm(const uint8_t *Aq, const uint8_t *As, const float *gA, const uint8_t *Wq,
                        const uint8_t *Ws, const float *gW, int64_t M, int64_t N, int64_t K,
                        int fmt, int bf16out, void *C, int64_t ldc, void *ws, size_t ws_bytes,
                        int sms, cudaStream_t st, int *timeout_flag_out, bool pdl, unsigned *counters,
                        bool w_before_wait);
cudaError_t launch_act_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, int fmt, int hk, float ck,
                                int round_away, int mx_floor, int gscale_given, uint8_t *q, uint8_t *s, float *gscale,
                                unsigned *zero, int nzero, int early, cudaStream_t st);
size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int fmt, int sms);
cudaError_t launch_gemm_quantized(const uint8_t *Aq, const uint8_t *As, const float *gA, const uint8_t *Wq,
                                  const uint8_t *Ws, const float *gW, int64_t M, int64_t N, int64_t K, int fmt,
                                  int out_fmt, int round_away, int mx_floor, const float *gC, uint8_t *Cq, uint8_t *Cs,
                                  int sms, cudaStream_t st);
cudaError_t launch_mx_to_nv_scales(const uint8_t *s_mx, int64_t rows, int64_t cols, uint8_t *s_nv, float *gscale,
                                   int sms, cudaStream_t st);
size_t nv_refine_workspace_bytes(int64_t rows, int64_t cols);
cudaError_t launch_nv_refine(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld, int hk, float ck,
                             int round_away, int rounds, uint8_t *q, uint8_t *s, void *ws, float *gscale, int sms,
                             cudaStream_t st);
cudaError_t launch_linear_fused(const uint16_t *x, int64_t ldx, int64_t M, int64_t K, int fmt, int hk, float ck,
                                int round_away, int mx_floor, const float *gA, const uint8_t *Wq, const uint8_t *Ws,
                                const float *gW, int64_t N, int bf16out, void *C, int64_t ldc, int sms, cudaStream_t st,
                                bool w_before_wait, bool residual, bool *taken);
cudaError_t read_and_clear_device_errors(cudaStream_t st, unsigned int *err);
static std::atomic<uint64_t> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }
}  // namespace fp4

namespace {

int sm_count()
{
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Format and block pairs of the quantizer; FP4_MXFP4 with block 16 is
// FP4_MXFP4_16 (norm_fmt).
bool valid_fmt(int fmt, int block)
{
    return (fmt == FP4_MXFP4 && (block == 32 || block == 16)) || (fmt == FP4_NVFP4 && block == 16) ||
           (fmt == FP4_MXFP4_16 && block == 16);
}

int norm_fmt(int fmt, int block) { return (fmt == FP4_MXFP4 && block == 16) ? FP4_MXFP4_16 : fmt; }

// Formats of the product (the block size follows from the format).
bool valid_gemm_fmt(int fmt) { return fmt == FP4_MXFP4 || fmt == FP4_NVFP4 || fmt == FP4_MXFP4_16; }

bool valid_k(int k) { return k == 0 || k == 16 || k == 32 || k == 64 || k == 128; }

// The streaming kernels index 32-element units with 32-bit integers: 2^32
// units are 2^37 elements, more than device memory holds as bf16.
bool too_many_units(int64_t rows, int64_t cols) { return cols > 0 && rows > ((int64_t(1) << 32) - 1) / (cols / 32 > 0 ? cols / 32 : 1); }

// RN_fp32(1/sqrt(k)): the double quotient is within 2^-52 relative of the
// exact value, far inside half an fp32 ulp, so rounding it once to fp32 gives
// the correctly rounded constant.
float hadamard_constant(int k) { return k ? (float)(1.0 / sqrt((double)k)) : 1.0f; }

}  // namespace

extern "C" {

const char *fp4_status_string(fp4_status st)
{
    switch (st) {
    case FP4_OK: return "FP4_OK";
    case FP4_ERR_INVALID_ARG: return "FP4_ERR_INVALID_ARG: invalid argument";
    case FP4_ERR_UNSUPPORTED: return "FP4_ERR_UNSUPPORTED: shape or format not supported";
    case FP4_ERR_ALIGNMENT: return "FP4_ERR_ALIGNMENT: pointer or stride misaligned";
    case FP4_ERR_CUDA: return "FP4_ERR_CUDA: CUDA runtime error";
    case FP4_ERR_TIMEOUT: return "FP4_ERR_TIMEOUT: a kernel gave up a bounded wait";
    }
    return "unknown fp4_status";
}

fp4_status fp4_quantize_sizes(int64_t rows, int64_t cols, int fmt, int block, size_t *q_bytes,
                              size_t *s_bytes)
{
    if (rows < 0 || cols < 0 || !q_bytes || !s_bytes) return FP4_ERR_INVALID_ARG;
    if (!valid_fmt(fmt, block)) return FP4_ERR_UNSUPPORTED;
    if (cols % block) return FP4_ERR_UNSUPPORTED;
    // byte counts must fit in 63 bits: rows * cols/2 and the padded scale tile
    if (rows > 0 && cols / 2 > (INT64_MAX - 127) / rows) return FP4_ERR_INVALID_ARG;
    const int64_t nkb = cols / block;
    if ((rows + 127) / 128 * 128 > 0 && (nkb + 3) / 4 * 4 > INT64_MAX / ((rows + 127) / 128 * 128))
        return FP4_ERR_INVALID_ARG;
    *q_bytes = (size_t)(rows * (cols / 2));
    *s_bytes = (size_t)(((rows + 127) / 128 * 128) * ((nkb + 3) / 4 * 4));
    return FP4_OK;
}

static fp4_status quantize_impl(const void *x, int64_t rows, int64_t cols, int64_t ld_x, int fmt, int block,
                                int hadamard_k, const fp4_opts *opts, uint8_t *q, uint8_t *s, float *gscale,
                                uint32_t *res, bool with_res, void *stream)
{
    fp4_opts o = {FP4_ROUND_EVEN, FP4_MX_SCALE_CEIL, 0, FP4_SCALE_ABSMAX, 0};
    if (opts) o = *opts;
    if (rows < 0 || cols < 0 || ld_x < cols) return FP4_ERR_INVALID_ARG;
    if (o.round != FP4_ROUND_EVEN && o.round != FP4_ROUND_AWAY) return FP4_ERR_INVALID_ARG;
    if (o.mx_scale_rule != FP4_MX_SCALE_CEIL && o.mx_scale_rule != FP4_MX_SCALE_FLOOR)
        return FP4_ERR_INVALID_ARG;
    if (o.scale_search != FP4_SCALE_ABSMAX && o.scale_search != FP4_SCALE_MSE) return FP4_ERR_INVALID_ARG;
    if (with_res && o.scale_search != FP4_SCALE_ABSMAX) return FP4_ERR_UNSUPPORTED;
    if (!valid_fmt(fmt, block) || !valid_k(hadamard_k)) return FP4_ERR_UNSUPPORTED;
    fmt = norm_fmt(fmt, block);
    if (cols % 32 || (hadamard_k && cols % hadamard_k)) return FP4_ERR_UNSUPPORTED;
    if (too_many_units(rows, cols)) return FP4_ERR_UNSUPPORTED;
    const bool empty = rows == 0 || cols == 0;
    if (fmt == FP4_NVFP4 && !gscale) return FP4_ERR_INVALID_ARG;
    if (!empty && (!x || !q || !s || (with_res && !res))) return FP4_ERR_INVALID_ARG;
    if (!aligned(x, 16) || (ld_x % 8) || !aligned(q, 16) || !aligned(s, 16)) return FP4_ERR_ALIGNMENT;
    if ((gscale && !aligned(gscale, 4)) || (res && !aligned(res, 4))) return FP4_ERR_ALIGNMENT;
    if (empty && fmt != FP4_NVFP4) return FP4_OK;
    cudaError_t e = fp4::launch_quantize(static_cast<const uint16_t *>(x), rows, cols, ld_x, fmt,
                                         hadamard_k, hadamard_constant(hadamard_k),
                                         o.round == FP4_ROUND_AWAY, o.mx_scale_rule == FP4_MX_SCALE_FLOOR,
                                         o.scale_search == FP4_SCALE_MSE, o.gscale_given, q, s, gscale, sm_count(),
                                         static_cast<cudaStream_t>(stream), true, with_res ? res : nullptr);
    return e == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
}

fp4_status fp4_quantize(const void *x, int64_t rows, int64_t cols, int64_t ld_x, int fmt, int block,
                        int hadamard_k, const fp4_opts *opts, uint8_t *q, uint8_t *s, float *gscale,
                        void *stream)
{
    return quantize_impl(x, rows, cols, ld_x, fmt, block, hadamard_k, opts, q, s, gscale, nullptr, false, stream);
}

fp4_status fp4_quantize_residual(const void *x, int64_t rows, int64_t cols, int64_t ld_x, int fmt, int block,
                                 int hadamard_k, const fp4_opts *opts, uint8_t *q, uint8_t *s, float *gscale,
                                 uint32_t *res, void *stream)
{
    return quantize_impl(x, rows, cols, ld_x, fmt, block, hadamard_k, opts, q, s, gscale, res, true, stream);
}

static fp4_status dequantize_impl(const uint8_t *q, const uint8_t *s, const float *gscale, const uint32_t *res,
                                  bool with_res, int64_t rows, int64_t cols, int fmt, int block, int hadamard_k,
                                  int out_dtype, void *out, void *stream)
{
    if (rows < 0 || cols < 0) return FP4_ERR_INVALID_ARG;
    if (out_dtype != FP4_OUT_F32 && out_dtype != FP4_OUT_BF16) return FP4_ERR_INVALID_ARG;
    if (!valid_fmt(fmt, block) || !valid_k(hadamard_k)) return FP4_ERR_UNSUPPORTED;
    fmt = norm_fmt(fmt, block);
    if (cols % 32 || (hadamard_k && cols % hadamard_k)) return FP4_ERR_UNSUPPORTED;
    if (too_many_units(rows, cols)) return FP4_ERR_UNSUPPORTED;
    if (rows == 0 || cols == 0) return FP4_OK;
    if (!q || !s || !out || (fmt == FP4_NVFP4 && !gscale) || (with_res && !res)) return FP4_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(s, 16) || !aligned(out, 16) || (res && !aligned(res, 4)))
        return FP4_ERR_ALIGNMENT;
    cudaError_t e = fp4::launch_dequantize(q, s, gscale, rows, cols, fmt, hadamard_k,
                                           hadamard_constant(hadamard_k), out_dtype == FP4_OUT_BF16,
                                           out, sm_count(), static_cast<cudaStream_t>(stream),
                                           with_res ? res : nullptr);
    return e == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
}

fp4_status fp4_dequantize(const uint8_t *q, const uint8_t *s, const float *gscale, int64_t rows,
                          int64_t cols, int fmt, int block, int hadamard_k, int out_dtype, void *out,
                          void *stream)
{
    return dequantize_impl(q, s, gscale, nullptr, false, rows, cols, fmt, block, hadamard_k, out_dtype, out,
                           stream);
}

fp4_status fp4_dequantize_residual(const uint8_t *q, const uint8_t *s, const float *gscale, const uint32_t *res,
                                   int64_t rows, int64_t cols, int fmt, int block, int hadamard_k, int out_dtype,
                                   void *out, void *stream)
{
    return dequantize_impl(q, s, gscale, res, true, rows, cols, fmt, block, hadamard_k, out_dtype, out, stream);
}

fp4_status fp4_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int fmt, size_t *bytes)
{
    if (M < 0 || N < 0 || K < 0 || !bytes) return FP4_ERR_INVALID_ARG;
    if (!valid_gemm_fmt(fmt)) return FP4_ERR_UNSUPPORTED;
    if (M > (1 << 30) || N > (1 << 30) || K > (1 << 30)) return FP4_ERR_UNSUPPORTED;  // as fp4_gemm
    *bytes = fp4::gemm_workspace_bytes(M, N, K, fmt, sm_count());
    return FP4_OK;
}

fp4_status fp4_gemm(const uint8_t *Aq, const uint8_t *As, const float *gA, const uint8_t *Wq,
                    const uint8_t *Ws, const float *gW, int64_t M, int64_t N, int64_t K, int fmt,
                    int out_dtype, void *C, int64_t ldc, void *workspace, size_t ws_bytes, void *stream)
{
    if (M < 0 || N < 0 || K < 0 || ldc < N) return FP4_ERR_INVALID_ARG;
    if (!valid_gemm_fmt(fmt)) return FP4_ERR_UNSUPPORTED;
    if (out_dtype != FP4_OUT_F32 && out_dtype != FP4_OUT_BF16) return FP4_ERR_INVALID_ARG;
    if (K % 32) return FP4_ERR_UNSUPPORTED;
    if (M == 0 || N == 0) return FP4_OK;
    if (!Aq || !As || !Wq || !Ws || !C) return FP4_ERR_INVALID_ARG;
    if (fmt == FP4_NVFP4 && (!gA || !gW)) return FP4_ERR_INVALID_ARG;
    if (!aligned(Aq, 16) || !aligned(Wq, 16) || !aligned(As, 16) || !aligned(Ws, 16) || !aligned(C, 16))
        return FP4_ERR_ALIGNMENT;
    const int sms = sm_count();
    const size_t need = fp4::gemm_workspace_bytes(M, N, K, fmt, sms);
    if (need > 0 && (!workspace || ws_bytes < need)) return FP4_ERR_INVALID_ARG;
    if (workspace && !aligned(workspace, 16)) return FP4_ERR_ALIGNMENT;
    int bad = 0;
    cudaError_t e = fp4::launch_gemm(Aq, As, gA, Wq, Ws, gW, M, N, K, fmt, out_dtype == FP4_OUT_BF16,
                                     C, ldc, workspace, ws_bytes, sms,
                                     static_cast<cudaStream_t>(stream), &bad, true, nullptr, false);
    if (bad) return FP4_ERR_UNSUPPORTED;
    return e == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
}

}  // extern "C"

namespace {
struct LinearLayout {
    size_t aq, as, ga, gemm, counters, total;
};

size_t round256(size_t b) { return (b + 255) / 256 * 256; }

LinearLayout linear_layout(int64_t M, int64_t N, int64_t K, int fmt, int sms)
{
    LinearLayout L;
    const int64_t nkb = K / (fmt == FP4_MXFP4 ? 32 : 16);
    L.aq = 0;
    L.as = round256((size_t)(M * (K / 2)));
    L.ga = L.as + round256((size_t)(((M + 127) / 128 * 128) * ((nkb + 3) / 4 * 4)));
    L.gemm = L.ga + 256;
    L.counters = L.gemm + round256(fp4::gemm_workspace_bytes(M, N, K, fmt, sms));
    // per-tile arrival counters of the decode kernel's fused reduction
    L.total = L.counters + round256((size_t)((N + 127) / 128) * sizeof(unsigned));
    return L;
}
}  // namespace

extern "C" {

fp4_status fp4_linear_workspace_size(int64_t M, int64_t N, int64_t K, int fmt, size_t *bytes)
{
    if (M < 0 || N < 0 || K < 0 || !bytes) return FP4_ERR_INVALID_ARG;
    if (!valid_gemm_fmt(fmt)) return FP4_ERR_UNSUPPORTED;
    if (M > (1 << 30) || N > (1 << 30) || K > (1 << 30)) return FP4_ERR_UNSUPPORTED;  // as fp4_gemm
    *bytes = linear_layout(M, N, K, fmt, sm_count()).total;
    return FP4_OK;
}

fp4_status fp4_linear(const void *x, int64_t M, int64_t K, int64_t ld_x, int fmt, int hadamard_k,
                      const fp4_opts *opts, const float *gA, const uint8_t *Wq, const uint8_t *Ws,
                      const float *gW, int64_t N, int out_dtype, void *C, int64_t ldc,
                      void *workspace, size_t ws_bytes, void *stream)
{
    fp4_opts o = {FP4_ROUND_EVEN, FP4_MX_SCALE_CEIL, 0, FP4_SCALE_ABSMAX, 0};
    if (opts) o = *opts;
    if (M < 0 || N < 0 || K < 0 || ld_x < K || ldc < N) return FP4_ERR_INVALID_ARG;
    if (!valid_gemm_fmt(fmt)) return FP4_ERR_UNSUPPORTED;
    if (out_dtype != FP4_OUT_F32 && out_dtype != FP4_OUT_BF16) return FP4_ERR_INVALID_ARG;
    if (o.round != FP4_ROUND_EVEN && o.round != FP4_ROUND_AWAY) return FP4_ERR_INVALID_ARG;
    if (o.mx_scale_rule != FP4_MX_SCALE_CEIL && o.mx_scale_rule != FP4_MX_SCALE_FLOOR) return FP4_ERR_INVALID_ARG;
    if (o.scale_search != FP4_SCALE_ABSMAX) return FP4_ERR_UNSUPPORTED;  // absmax scales only
    if (o.weights_static != 0 && o.weights_static != 1) return FP4_ERR_INVALID_ARG;
    if (!valid_k(hadamard_k)) return FP4_ERR_UNSUPPORTED;
    if (K % 32 || (hadamard_k && K % hadamard_k)) return FP4_ERR_UNSUPPORTED;
    if (too_many_units(M, K)) return FP4_ERR_UNSUPPORTED;
    if (M > (1 << 30) || N > (1 << 30) || K > (1 << 30)) return FP4_ERR_UNSUPPORTED;  // as fp4_gemm
    if (M == 0 || N == 0) return FP4_OK;
    if (!x || !Wq || !Ws || !C || !workspace) return FP4_ERR_INVALID_ARG;
    if (fmt == FP4_NVFP4 && !gW) return FP4_ERR_INVALID_ARG;
    if (!aligned(x, 16) || (ld_x % 8) || !aligned(Wq, 16) || !aligned(Ws, 16) || !aligned(C, 16) ||
        !aligned(workspace, 256))
        return FP4_ERR_ALIGNMENT;
    const int sms = sm_count();
    const LinearLayout L = linear_layout(M, N, K, fmt, sms);
    if (ws_bytes < L.total) return FP4_ERR_INVALID_ARG;
    uint8_t *base = static_cast<uint8_t *>(workspace);
    uint8_t *aq = base + L.aq, *as = base + L.as;
    float *ga = (fmt == FP4_NVFP4 && gA) ? const_cast<float *>(gA) : reinterpret_cast<float *>(base + L.ga);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool decode = M <= 16;
    unsigned *counters = decode ? reinterpret_cast<unsigned *>(base + L.counters) : nullptr;
    cudaError_t e;
    if (decode) {
        // one launch: the decode kernel quantizes the activations itself
        // (whole-tile and cluster work splits)
        bool taken = false;
        e = fp4::launch_linear_fused(static_cast<const uint16_t *>(x), ld_x, M, K, fmt, hadamard_k,
                                     hadamard_constant(hadamard_k), o.round == FP4_ROUND_AWAY,
                                     o.mx_scale_rule == FP4_MX_SCALE_FLOOR, fmt == FP4_NVFP4 ? gA : nullptr, Wq, Ws, gW,
                                     N, out_dtype == FP4_OUT_BF16, C, ldc, sms, st, o.weights_static != 0, false,
                                     &taken);
        if (taken) return e == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
        // otherwise two launches: one cluster quantizes the activations (and
        // zeroes the tile counters); the split-K kernel streams W meanwhile
        // and reduces.
        e = fp4::launch_act_quantize(static_cast<const uint16_t *>(x), M, K, ld_x, fmt, hadamard_k,
                                     hadamard_constant(hadamard_k), o.round == FP4_ROUND_AWAY,
                                     o.mx_scale_rule == FP4_MX_SCALE_FLOOR, gA != nullptr, aq, as, ga, counters,
                                     (int)((N + 127) / 128), o.weights_static != 0, st);
    } else {
        e = fp4::launch_quantize(static_cast<const uint16_t *>(x), M, K, ld_x, fmt, hadamard_k,
                                 hadamard_constant(hadamard_k), o.round == FP4_ROUND_AWAY,
                                 o.mx_scale_rule == FP4_MX_SCALE_FLOOR, 0, gA != nullptr, aq, as, ga, sms, st, true,
                                 nullptr);
    }
    if (e != cudaSuccess) return FP4_ERR_CUDA;
    int bad = 0;
    e = fp4::launch_gemm(aq, as, ga, Wq, Ws, gW, M, N, K, fmt, out_dtype == FP4_OUT_BF16, C, ldc, base + L.gemm,
                         L.counters - L.gemm, sms, st, &bad, true, counters, decode);
    if (bad) return FP4_ERR_UNSUPPORTED;
    return e == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
}

fp4_status fp4_linear_residual(const void *x, int64_t M, int64_t K, int64_t ld_x, int fmt, int hadamard_k,
                               const fp4_opts *opts, const float *gA, const uint8_t *Wq, const uint8_t *Ws,
                               const float *gW, int64_t N, int out_dtype, void *C, int64_t ldc, void *stream)
{
    fp4_opts o = {FP4_ROUND_EVEN, FP4_MX_SCALE_CEIL, 0, FP4_SCALE_ABSMAX, 0};
    if (opts) o = *opts;
    if (M < 0 || N < 0 || K < 0 || ld_x < K || ldc < N) return FP4_ERR_INVALID_ARG;
    if (!valid_gemm_fmt(fmt)) return FP4_ERR_UNSUPPORTED;
    if (out_dtype != FP4_OUT_F32 && out_dtype != FP4_OUT_BF16) return FP4_ERR_INVALID_ARG;
    if (o.round != FP4_ROUND_EVEN && o.round != FP4_ROUND_AWAY) return FP4_ERR_INVALID_ARG;
    if (o.mx_scale_rule != FP4_MX_SCALE_CEIL && o.mx_scale_rule != FP4_MX_SCALE_FLOOR) return FP4_ERR_INVALID_ARG;
    if (o.scale_search != FP4_SCALE_ABSMAX) return FP4_ERR_UNSUPPORTED;
    if (o.weights_static != 0 && o.weights_static != 1) return FP4_ERR_INVALID_ARG;
    if (!valid_k(hadamard_k)) return FP4_ERR_UNSUPPORTED;
    if (K % 32 || (hadamard_k && K % hadamard_k)) return FP4_ERR_UNSUPPORTED;
    if (M > 16 || N > (1 << 30) || K > (1 << 30)) return FP4_ERR_UNSUPPORTED;  // the decode product only
    if (M == 0 || N == 0) return FP4_OK;
    if (K == 0) return FP4_ERR_UNSUPPORTED;
    if (!x || !Wq || !Ws || !C) return FP4_ERR_INVALID_ARG;
    if (fmt == FP4_NVFP4 && !gW) return FP4_ERR_INVALID_ARG;
    if (!aligned(x, 16) || (ld_x % 8) || !aligned(Wq, 16) || !aligned(Ws, 16) || !aligned(C, 16))
        return FP4_ERR_ALIGNMENT;
    if (gA && !aligned(gA, 4)) return FP4_ERR_ALIGNMENT;
    bool taken = false;
    const cudaError_t e = fp4::launch_linear_fused(
        static_cast<const uint16_t *>(x), ld_x, M, K, fmt, hadamard_k, hadamard_constant(hadamard_k),
        o.round == FP4_ROUND_AWAY, o.mx_scale_rule == FP4_MX_SCALE_FLOOR, fmt == FP4_NVFP4 ? gA : nullptr, Wq, Ws, gW,
        N, out_dtype == FP4_OUT_BF16, C, ldc, sm_count(), static_cast<cudaStream_t>(stream), o.weights_static != 0, true,
        &taken);
    if (!taken) return FP4_ERR_UNSUPPORTED;
    return e == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
}

fp4_status fp4_gemm_quantized(const uint8_t *Aq, const uint8_t *As, const float *gA, const uint8_t *Wq,
                              const uint8_t *Ws, const float *gW, int64_t M, int64_t N, int64_t K, int fmt,
                              int out_fmt, const fp4_opts *opts, const float *gC, uint8_t *Cq, uint8_t *Cs,
                              void *stream)
{
    fp4_opts o = {FP4_ROUND_EVEN, FP4_MX_SCALE_CEIL, 0, FP4_SCALE_ABSMAX, 0};
    if (opts) o = *opts;
    if (M < 0 || N < 0 || K < 0) return FP4_ERR_INVALID_ARG;
    if (!valid_gemm_fmt(fmt)) return FP4_ERR_UNSUPPORTED;
    if (out_fmt != FP4_MXFP4 && out_fmt != FP4_NVFP4) return FP4_ERR_UNSUPPORTED;
    if (o.round != FP4_ROUND_EVEN && o.round != FP4_ROUND_AWAY) return FP4_ERR_INVALID_ARG;
    if (o.mx_scale_rule != FP4_MX_SCALE_CEIL && o.mx_scale_rule != FP4_MX_SCALE_FLOOR) return FP4_ERR_INVALID_ARG;
    if (o.scale_search != FP4_SCALE_ABSMAX) return FP4_ERR_UNSUPPORTED;  // absmax scales only
    if (M <= 16 || K % 32 || N % 128) return FP4_ERR_UNSUPPORTED;
    if (M > (1 << 30) || N > (1 << 30) || K > (1 << 30)) return FP4_ERR_UNSUPPORTED;
    if (!Aq || !As || !Wq || !Ws || !Cq || !Cs) return FP4_ERR_INVALID_ARG;
    if (fmt == FP4_NVFP4 && (!gA || !gW)) return FP4_ERR_INVALID_ARG;
    if (out_fmt == FP4_NVFP4 && !gC) return FP4_ERR_INVALID_ARG;
    if (!aligned(Aq, 16) || !aligned(Wq, 16) || !aligned(As, 16) || !aligned(Ws, 16) || !aligned(Cq, 16) ||
        !aligned(Cs, 16))
        return FP4_ERR_ALIGNMENT;
    if (gC && !aligned(gC, 4)) return FP4_ERR_ALIGNMENT;
    cudaError_t e = fp4::launch_gemm_quantized(Aq, As, gA, Wq, Ws, gW, M, N, K, fmt, out_fmt,
                                               o.round == FP4_ROUND_AWAY, o.mx_scale_rule == FP4_MX_SCALE_FLOOR,
                                               gC, Cq, Cs, sm_count(), static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
}

fp4_status fp4_mx_to_nv_scales(const uint8_t *s_mx, int64_t rows, int64_t cols, uint8_t *s_nv, float *gscale,
                               void *stream)
{
    if (rows < 0 || cols < 0 || !gscale) return FP4_ERR_INVALID_ARG;
    if (cols % 32) return FP4_ERR_UNSUPPORTED;
    if (too_many_units(rows, cols)) return FP4_ERR_UNSUPPORTED;
    if (rows > 0 && cols > 0 && (!s_mx || !s_nv)) return FP4_ERR_INVALID_ARG;
    if (!aligned(gscale, 4)) return FP4_ERR_ALIGNMENT;
    cudaError_t e = fp4::launch_mx_to_nv_scales(s_mx, rows, cols, s_nv, gscale, sm_count(),
                                                static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
}

fp4_status fp4_nv_refine_gscale_workspace_size(int64_t rows, int64_t cols, size_t *bytes)
{
    if (rows < 0 || cols < 0 || !bytes) return FP4_ERR_INVALID_ARG;
    if (cols % 32) return FP4_ERR_UNSUPPORTED;
    *bytes = fp4::nv_refine_workspace_bytes(rows, cols);
    return FP4_OK;
}

fp4_status fp4_nv_refine_gscale(const void *x, int64_t rows, int64_t cols, int64_t ld_x, int hadamard_k,
                                const fp4_opts *opts, int rounds, uint8_t *q, uint8_t *s, void *workspace,
                                size_t ws_bytes, float *gscale, void *stream)
{
    fp4_opts o = {FP4_ROUND_EVEN, FP4_MX_SCALE_CEIL, 0, FP4_SCALE_ABSMAX, 0};
    if (opts) o = *opts;
    if (rows < 0 || cols < 0 || ld_x < cols || rounds < 1 || rounds > 64) return FP4_ERR_INVALID_ARG;
    if (o.round != FP4_ROUND_EVEN && o.round != FP4_ROUND_AWAY) return FP4_ERR_INVALID_ARG;
    if (!valid_k(hadamard_k)) return FP4_ERR_UNSUPPORTED;
    if (cols % 32 || (hadamard_k && cols % hadamard_k)) return FP4_ERR_UNSUPPORTED;
    if (too_many_units(rows, cols)) return FP4_ERR_UNSUPPORTED;
    if (!gscale || !workspace) return FP4_ERR_INVALID_ARG;
    if (rows > 0 && cols > 0 && (!x || !q || !s)) return FP4_ERR_INVALID_ARG;
    if (!aligned(x, 16) || (ld_x % 8) || !aligned(q, 16) || !aligned(s, 16) || !aligned(workspace, 256) ||
        !aligned(gscale, 4))
        return FP4_ERR_ALIGNMENT;
    if (ws_bytes < fp4::nv_refine_workspace_bytes(rows, cols)) return FP4_ERR_INVALID_ARG;
    cudaError_t e = fp4::launch_nv_refine(static_cast<const uint16_t *>(x), rows, cols, ld_x, hadamard_k,
                                          hadamard_constant(hadamard_k), o.round == FP4_ROUND_AWAY, rounds, q, s,
                                          workspace, gscale, sm_count(), static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? FP4_OK : FP4_ERR_CUDA;
}

uint64_t fp4_kernel_launches(void) { return fp4::g_launches.load(std::memory_order_relaxed); }

fp4_status fp4_check_device_status(void *stream)
{
    unsigned int err = 0;
    if (fp4::read_and_clear_device_errors(static_cast<cudaStream_t>(stream), &err) != cudaSuccess)
        return FP4_ERR_CUDA;
    return err ? FP4_ERR_TIMEOUT : FP4_OK;
}

}  // extern "C"
