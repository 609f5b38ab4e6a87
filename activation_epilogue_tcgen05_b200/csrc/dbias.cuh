// dbias.cuh -- bias-gradient reductions for the ReLU backward epilogue.
//
// The backward of z = alpha*A.B + bias, y = relu(z) needs dbias, the sum of
// dz over the axis the bias was broadcast along ("nvmath-python cuBLASLt bias
// fusion for PyTorch inference" (blog.hotdry.top), paragraphs 6-7: the aux
// mask exists for the backward pass, and fusing dBias is the next step).
//
//   sum_parts_kernel  out[i] = sum_{p < parts} src[p * len + i], p in increasing
//                     order.  Fused path: src = the fp32 partials the GEMM's
//                     epilogue wrote.  Unfused path, COL axis: src = D itself
//                     (parts = m rows, len = n).
//   sum_rows_kernel   out[i] = sum_j D[i, j] (unfused path, ROW axis), one warp
//                     per row, lane-strided then a fixed xor-butterfly.
//
// Every sum is taken in fp32 in an order fixed by the shapes alone, so results
// are identical from run to run; the result is rounded once to the bias type.
#pragma once
#include <cstdint>

#include "gemm_tc.cuh"

namespace gemm_epi {

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__half>(__half x) { return __half2float(x); }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <int DT>
__device__ __forceinline__ void store_out(void *out, int64_t i, float v) {
    if constexpr (DT == DT_F16) reinterpret_cast<__half *>(out)[i] = __float2half_rn(v);
    else reinterpret_cast<__nv_bfloat16 *>(out)[i] = __float2bfloat16_rn(v);
}

// Block: 32 consecutive outputs x SUM_PARTS_Y part-strides.  Thread (x, y) sums
// parts y, y + Y, y + 2Y, ... of output x into four independent accumulators (so
// four loads are in flight), combines them in a fixed order, and row y = 0 then adds
// the Y strides in order: the result depends only on (parts, len).
constexpr int SUM_PARTS_Y = 32;

template <typename IN, int DT>
__global__ void __launch_bounds__(32 * SUM_PARTS_Y) sum_parts_kernel(const IN *__restrict__ src, int64_t parts,
                                                                  int64_t len, void *out) {
    __shared__ float red[SUM_PARTS_Y][33];
    // launched as a dependent of the kernel that wrote src: wait for it before reading;
    // the next kernel (itself waiting before any global access) may then be scheduled
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int64_t i = (int64_t)blockIdx.x * 32 + threadIdx.x;
    float s = 0.0f;
    if (i < len) {
        constexpr int Y = SUM_PARTS_Y;
        float s0 = 0.0f, s1 = 0.0f, s2 = 0.0f, s3 = 0.0f;
        int64_t p = threadIdx.y;
        for (; p + 3 * Y < parts; p += 4 * Y) {
            s0 += to_f32(__ldg(src + p * len + i));
            s1 += to_f32(__ldg(src + (p + Y) * len + i));
            s2 += to_f32(__ldg(src + (p + 2 * Y) * len + i));
            s3 += to_f32(__ldg(src + (p + 3 * Y) * len + i));
        }
        for (; p < parts; p += Y) s0 += to_f32(__ldg(src + p * len + i));
        s = (s0 + s1) + (s2 + s3);
    }
    red[threadIdx.y][threadIdx.x] = s;
    __syncthreads();
    if (threadIdx.y == 0 && i < len) {
        float t = red[0][threadIdx.x];
#pragma unroll
        for (int y = 1; y < SUM_PARTS_Y; ++y) t += red[y][threadIdx.x];
        store_out<DT>(out, i, t);
    }
}

// One warp per row of a row-major (m, n) 16-bit matrix; n is a multiple of 8.
template <int DT>
__global__ void __launch_bounds__(256) sum_rows_kernel(const void *__restrict__ D, int64_t m, int64_t n, void *out) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
    using T = typename OutT<DT>::type;
    for (int64_t i = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32; i < m; i += warps) {
        const T *row = reinterpret_cast<const T *>(D) + i * n;
        float s = 0.0f;
        for (int64_t j = (int64_t)lane * 8; j < n; j += 256) {
            float f[8];
            unpack8<DT == DT_F16 ? DT_F16 : DT_BF16>(__ldg(reinterpret_cast<const uint4 *>(row + j)), f);
#pragma unroll
            for (int e = 0; e < 8; ++e) s += f[e];
        }
#pragma unroll
        for (int sh = 16; sh >= 1; sh >>= 1) s += __shfl_xor_sync(0xffffffffu, s, sh);
        if (lane == 0) store_out<DT>(out, i, s);
    }
}

}  // namespace gemm_epi
