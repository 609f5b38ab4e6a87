// quant.cuh -- the UNFUSED form of the FP8 requantisation of an MLP block's
// intermediate: after a GEMM has written H in bf16 and a separate kernel has
// applied bias and activation, one pass finds amax = max |H| and another stores
// e4m3(H / s_H).  This is the sequence the requantising epilogue replaces; it
// is kept as the library's own baseline for time and traffic comparisons.
#pragma once
#include <cstdint>

#include "gemm_tc.cuh"

namespace gemm_epi {

// max |x| over `count` bf16 values (count a multiple of 8, x 16-byte aligned), max-reduced
// into *amax as float bits: non-negative floats order as their bit patterns, so the result
// does not depend on the order of the atomics.
__global__ void __launch_bounds__(256) amax_bf16_kernel(const void *__restrict__ x, int64_t count,
                                                        unsigned int *amax) {
    const uint4 *v = reinterpret_cast<const uint4 *>(x);
    float m = 0.0f;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < count / 8;
         i += (int64_t)gridDim.x * blockDim.x) {
        float f[8];
        unpack8<DT_BF16>(__ldg(v + i), f);
#pragma unroll
        for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(f[e]));
    }
    const unsigned int w = __reduce_max_sync(0xffffffffu, __float_as_uint(m));
    if ((threadIdx.x & 31) == 0) atomicMax(amax, w);
}

// q[i] = e4m3(x[i] / *scale), round to nearest even, saturating at +-448; 8 values a thread step.
__global__ void __launch_bounds__(256) quantize_bf16_e4m3_kernel(const void *__restrict__ x, int64_t count,
                                                                 const float *__restrict__ scale, uint8_t *q) {
    const uint4 *v = reinterpret_cast<const uint4 *>(x);
    uint2 *out = reinterpret_cast<uint2 *>(q);
    const float inv = 1.0f / __ldg(scale);
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < count / 8;
         i += (int64_t)gridDim.x * blockDim.x) {
        float f[8];
        unpack8<DT_BF16>(__ldg(v + i), f);
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
            w[e] = __nv_cvt_float2_to_fp8x2(make_float2(f[2 * e] * inv, f[2 * e + 1] * inv), __NV_SATFINITE, __NV_E4M3);
        out[i] = make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
    }
}

}  // namespace gemm_epi
