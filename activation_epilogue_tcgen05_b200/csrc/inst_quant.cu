// Launchers of the unfused requantisation kernels (quant.cuh).
#include "kernels.h"
#include "quant.cuh"

namespace gemm_epi {

cudaError_t launch_amax_bf16(const void *x, int64_t count, unsigned int *amax, int grid, cudaStream_t s) {
    if (count <= 0) return cudaSuccess;
    amax_bf16_kernel<<<grid, 256, 0, s>>>(x, count, amax);
    return cudaGetLastError();
}

cudaError_t launch_quantize_bf16_e4m3(const void *x, int64_t count, const float *scale, uint8_t *q, int grid,
                                      cudaStream_t s) {
    if (count <= 0) return cudaSuccess;
    quantize_bf16_e4m3_kernel<<<grid, 256, 0, s>>>(x, count, scale, q);
    return cudaGetLastError();
}

}  // namespace gemm_epi
