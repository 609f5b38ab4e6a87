// bias_act.cuh -- the UNFUSED second step: read the bare GEMM's output back
// from HBM, add the bias, apply the activation, write D (in place) and the
// sign mask.  This is the stepwise sequence the fused kernel replaces
// ("nvmath-python epilog bias fusion parameters" (blog.hotdry.top), body
// paragraph 1: matmul, write back, separate element-wise kernel), kept as the
// library's own baseline for time and DRAM-traffic comparisons.
//
// EPI_DRELU is the backward step of the same baseline: it reads the packed mask
// from aux and zeroes D where the mask bit is 0 (no bias).
//
// One thread owns 32 consecutive columns of one row -- exactly one 32-bit
// mask word -- and moves them with four 16-byte loads and stores; consecutive
// threads take consecutive words of a row, so a warp streams 2 KB contiguous.
#pragma once
#include <cstdint>

#include "gemm_tc.cuh"

namespace gemm_epi {

template <int DT, int EPI, int AXIS>
__global__ void __launch_bounds__(256) bias_act_kernel(void *D, const void *bias, uint32_t *aux,
                                                       int m, int n, int64_t pitch_words,
                                                       int64_t total_words) {
    using O = OutT<DT>;
    using T = typename O::type;
    T *d = reinterpret_cast<T *>(D);
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total_words;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = idx / pitch_words;
        const int64_t w = idx - i * pitch_words;
        const int j0 = (int)(w * 32);
        if (j0 >= n) {                     // padding word of the mask row
            if constexpr (EPI == EPI_RELU_AUX) aux[idx] = 0u;
            continue;
        }
        T *row = d + i * (int64_t)n;
        float rb = 0.0f;
        if constexpr (AXIS == AXIS_ROW) {
            if (bias != nullptr) rb = O::load(bias, i);
        }
        uint32_t bits = 0;
        uint32_t mbits = 0;
        if constexpr (EPI == EPI_DRELU) mbits = aux[idx];
        if (j0 + 32 <= n) {
            uint4 *src = reinterpret_cast<uint4 *>(row + j0);
            uint4 u[4];
#pragma unroll
            for (int s = 0; s < 4; ++s) u[s] = src[s];
            float bcol[32];
            if constexpr (AXIS == AXIS_COL) if (bias == nullptr) {
#pragma unroll
                for (int e = 0; e < 32; ++e) bcol[e] = 0.0f;
            } else {
                const uint4 *bsrc = reinterpret_cast<const uint4 *>(reinterpret_cast<const T *>(bias) + j0);
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    float f[8];
                    unpack8<DT == DT_F16 ? DT_F16 : DT_BF16>(__ldg(bsrc + s), f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) bcol[8 * s + e] = f[e];
                }
            }
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                float f[8];
                unpack8<DT == DT_F16 ? DT_F16 : DT_BF16>(u[s], f);
                uint32_t outw[4];
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    float x0 = f[e] + (AXIS == AXIS_ROW ? rb : bcol[8 * s + e]);
                    float x1 = f[e + 1] + (AXIS == AXIS_ROW ? rb : bcol[8 * s + e + 1]);
                    if constexpr (EPI == EPI_DRELU) {
                        x0 = ((mbits >> (8 * s + e)) & 1u) ? f[e] : 0.0f;
                        x1 = ((mbits >> (8 * s + e + 1)) & 1u) ? f[e + 1] : 0.0f;
                    }
                    if constexpr (EPI == EPI_RELU_AUX) {
                        bits |= (x0 > 0.0f ? 1u : 0u) << (8 * s + e);
                        bits |= (x1 > 0.0f ? 1u : 0u) << (8 * s + e + 1);
                    }
                    outw[e / 2] = O::pack(activate<EPI>(x0), activate<EPI>(x1));
                }
                src[s] = make_uint4(outw[0], outw[1], outw[2], outw[3]);
            }
        } else {
            for (int j = j0; j < n; ++j) {
                float x = O::load(row, j) + (AXIS == AXIS_ROW ? rb : (bias != nullptr ? O::load(bias, j) : 0.0f));
                if constexpr (EPI == EPI_DRELU) x = ((mbits >> (j - j0)) & 1u) ? O::load(row, j) : 0.0f;
                if constexpr (EPI == EPI_RELU_AUX) bits |= (x > 0.0f ? 1u : 0u) << (j - j0);
                const float y = activate<EPI>(x);
                if constexpr (DT == DT_F16) row[j] = __float2half_rn(y);
                else row[j] = __float2bfloat16_rn(y);
            }
        }
        if constexpr (EPI == EPI_RELU_AUX) aux[idx] = bits;
    }
}

}  // namespace gemm_epi
