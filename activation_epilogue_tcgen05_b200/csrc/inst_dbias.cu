// Instantiations of the bias-gradient reductions (dbias.cuh).
#include "dbias.cuh"
#include "kernels.h"

namespace gemm_epi {

namespace {
template <typename IN>
cudaError_t sum_parts(int out_dt, const IN *src, int64_t parts, int64_t len, void *out, bool pdl, cudaStream_t s) {
    if (len <= 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((len + 31) / 32), 1, 1);
    cfg.blockDim = dim3(32, SUM_PARTS_Y, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    if (pdl) {     // its launch overlaps the tail of the kernel that writes src
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    if (out_dt == DT_F16) return cudaLaunchKernelEx(&cfg, sum_parts_kernel<IN, DT_F16>, src, parts, len, out);
    return cudaLaunchKernelEx(&cfg, sum_parts_kernel<IN, DT_BF16>, src, parts, len, out);
}
}  // namespace

cudaError_t launch_sum_parts_f32(int out_dt, const float *src, int64_t parts, int64_t len, void *out, bool pdl,
                                 cudaStream_t s) {
    return sum_parts<float>(out_dt, src, parts, len, out, pdl, s);
}

cudaError_t launch_sum_cols(int out_dt, const void *D, int64_t m, int64_t n, void *out, cudaStream_t s) {
    if (out_dt == DT_F16) return sum_parts<__half>(out_dt, reinterpret_cast<const __half *>(D), m, n, out, false, s);
    return sum_parts<__nv_bfloat16>(out_dt, reinterpret_cast<const __nv_bfloat16 *>(D), m, n, out, false, s);
}

cudaError_t launch_sum_rows(int out_dt, const void *D, int64_t m, int64_t n, void *out, int grid, cudaStream_t s) {
    if (m <= 0) return cudaSuccess;
    if (out_dt == DT_F16) sum_rows_kernel<DT_F16><<<grid, 256, 0, s>>>(D, m, n, out);
    else sum_rows_kernel<DT_BF16><<<grid, 256, 0, s>>>(D, m, n, out);
    return cudaGetLastError();
}

}  // namespace gemm_epi
