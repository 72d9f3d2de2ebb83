// gemm.cu — block-scaled W4A4 GEMM kernels (placeholder until the tcgen05
// kernels land: every call reports the shape as unsupported).
#include "common.cuh"

namespace fp4 {

static __device__ unsigned int g_gemm_error;

size_t gemm_workspace_bytes(int64_t, int64_t, int64_t, int, int) { return 0; }

cudaError_t launch_gemm(const uint8_t *, const uint8_t *, const float *, const uint8_t *,
                        const uint8_t *, const float *, int64_t, int64_t, int64_t, int, int,
                        void *, int64_t, void *, size_t, int, cudaStream_t, int *bad)
{
    *bad = 1;
    return cudaSuccess;
}

cudaError_t read_and_clear_device_errors(cudaStream_t st, unsigned int *err)
{
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return e;
    unsigned int v = 0;
    if ((e = cudaMemcpyFromSymbol(&v, g_gemm_error, sizeof v)) != cudaSuccess) return e;
    const unsigned int zero = 0;
    if ((e = cudaMemcpyToSymbol(g_gemm_error, &zero, sizeof zero)) != cudaSuccess) return e;
    *err = v;
    return cudaSuccess;
}

}  // namespace fp4
