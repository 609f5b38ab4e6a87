// kernels.h -- internal interface between the C-ABI layer (gemm_epi_api.cu)
// and the kernel instantiation units (inst_*.cu).  Not installed, not public.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "gemm_splitk.cuh"
#include "gemm_splitk_grid.cuh"
#include "gemm_tc.cuh"

namespace gemm_epi {

// One persistent tcgen05 launch.
struct TcLaunch {
    CUtensorMap tmA, tmB, tmD;
    TcParams p;
    int grid;
    bool pdl;            // launch with programmatic stream serialisation
    cudaStream_t stream;
};
// One split-K cluster launch.
struct SkLaunch {
    CUtensorMap tmW, tmX;
    SkParams p;
    int grid;
    int cluster;
    bool pdl;            // launch with programmatic stream serialisation
    cudaStream_t stream;
};

// One grid-wide split-K launch (no cluster).
struct SgLaunch {
    CUtensorMap tmW, tmX;
    SgParams p;
    bool pdl;            // launch with programmatic stream serialisation
    cudaStream_t stream;
};

struct KernelInfo {
    const void *func;   // the __global__ symbol (for attributes / occupancy queries)
    int threads;
    int smem_bytes;
    int stages;
    int block_m, block_n, block_k;   // block_k: k per ring stage
    int katoms = 1;                  // 128-byte k-atoms per ring stage
};

using TcLauncher = cudaError_t (*)(const TcLaunch &);
using SkLauncher = cudaError_t (*)(const SkLaunch &);
using SgLauncher = cudaError_t (*)(const SgLaunch &);
using BiasActLauncher = cudaError_t (*)(void *D, const void *bias, uint32_t *aux, int m, int n,
                                        int64_t pitch_words, int grid, cudaStream_t stream);

// Lookups return false when the combination is not instantiated.
// qout: e4m3 output quantised in the epilogue (e4m3 operands only); a_mn: A stored (k, m)
bool find_tc(int cg, int dt, int epi, int axis, bool b_mn, int bn, bool qout, bool a_mn, TcLauncher *launch,
             KernelInfo *info);
bool find_sk(int dt, int epi, int axis, bool w_mn, int nm, bool qout, SkLauncher *launch, KernelInfo *info);
bool find_sg(int dt, int epi, int axis, bool w_mn, int nm, bool qout, SgLauncher *launch, KernelInfo *info);
bool find_bias_act(int dt, int epi, int axis, BiasActLauncher *launch);

// Bias-gradient reductions (dbias.cuh); out_dt is the bias type (DT_F16 or DT_BF16).
//   sum_parts_f32: out[i] = sum_p src[p * len + i] over fp32 partials (fused backward)
//   sum_cols:      out[j] = sum_i D[i, j]  (unfused backward, COL axis)
//   sum_rows:      out[i] = sum_j D[i, j]  (unfused backward, ROW axis)
cudaError_t launch_sum_parts_f32(int out_dt, const float *src, int64_t parts, int64_t len, void *out, bool pdl,
                                 cudaStream_t s);
cudaError_t launch_sum_cols(int out_dt, const void *D, int64_t m, int64_t n, void *out, cudaStream_t s);
cudaError_t launch_sum_rows(int out_dt, const void *D, int64_t m, int64_t n, void *out, int grid, cudaStream_t s);

// The unfused requantisation (quant.cuh): amax of a bf16 array (count a multiple of 8) into
// float bits, and its e4m3 quantisation with a device scale.
cudaError_t launch_amax_bf16(const void *x, int64_t count, unsigned int *amax, int grid, cudaStream_t s);
cudaError_t launch_quantize_bf16_e4m3(const void *x, int64_t count, const float *scale, uint8_t *q, int grid,
                                      cudaStream_t s);

// per-dtype halves of the lookups (one instantiation unit each)
bool find_tc_f16(int cg, int epi, int axis, bool b_mn, int bn, TcLauncher *, KernelInfo *);
bool find_tc_bf16(int cg, int epi, int axis, bool b_mn, int bn, TcLauncher *, KernelInfo *);
bool find_tc_e4m3(int cg, int epi, int axis, bool b_mn, int bn, TcLauncher *, KernelInfo *);
bool find_tc_e4m3_q(int cg, int epi, int axis, bool b_mn, int bn, TcLauncher *, KernelInfo *);
bool find_tc_f16_at(int cg, int epi, int axis, bool b_mn, int bn, TcLauncher *, KernelInfo *);
bool find_tc_bf16_at(int cg, int epi, int axis, bool b_mn, int bn, TcLauncher *, KernelInfo *);
bool find_tc_e4m3_at(int cg, int epi, int axis, bool b_mn, int bn, TcLauncher *, KernelInfo *);
bool find_sk_f16(int epi, int axis, bool w_mn, int nm, SkLauncher *, KernelInfo *);
bool find_sk_bf16(int epi, int axis, bool w_mn, int nm, SkLauncher *, KernelInfo *);
bool find_sk_e4m3(int epi, int axis, bool w_mn, int nm, SkLauncher *, KernelInfo *);
bool find_sk_e4m3_q(int epi, int axis, bool w_mn, int nm, SkLauncher *, KernelInfo *);
bool find_sg_f16(int epi, int axis, bool w_mn, int nm, SgLauncher *, KernelInfo *);
bool find_sg_bf16(int epi, int axis, bool w_mn, int nm, SgLauncher *, KernelInfo *);
bool find_sg_e4m3(int epi, int axis, bool w_mn, int nm, SgLauncher *, KernelInfo *);
bool find_sg_e4m3_q(int epi, int axis, bool w_mn, int nm, SgLauncher *, KernelInfo *);

// Ring depth that fills GEMM_EPI_RING_KB (default 192) KB of shared memory with stages.
#ifndef GEMM_EPI_RING_KB
#define GEMM_EPI_RING_KB 192
#endif
constexpr int tc_stages(int stage_bytes) { return (GEMM_EPI_RING_KB * 1024) / stage_bytes; }

// Shared launch helpers used by the instantiation units.
template <class C>
cudaError_t launch_tc(const TcLaunch &L) {
    auto kern = tc_gemm_kernel<C>;
    static int attr_done[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_done[dev] = 1;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(L.grid, 1, 1);
    cfg.blockDim = dim3(C::THREADS, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = L.stream;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if constexpr (C::CG == 2) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = 2;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    if (L.pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = na ? attr : nullptr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, kern, L.tmA, L.tmB, L.tmD, L.p);
}

template <class C>
KernelInfo tc_info() {
    KernelInfo k;
    k.func = reinterpret_cast<const void *>(tc_gemm_kernel<C>);
    k.threads = C::THREADS;
    k.smem_bytes = C::SMEM_BYTES;
    k.stages = C::STAGES;
    k.block_m = C::BM * C::CG;
    k.block_n = C::BN;
    k.block_k = C::BK * C::KATOMS;
    k.katoms = C::KATOMS;
    return k;
}

template <class C>
cudaError_t launch_sk(const SkLaunch &L) {
    auto kern = splitk_gemm_kernel<C>;
    static int attr_done[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_done[dev] = 1;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(L.grid, 1, 1);
    cfg.blockDim = dim3(C::THREADS, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = L.stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = L.cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    int na = 1;
    if (L.pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, kern, L.tmW, L.tmX, L.p);
}

template <class C>
KernelInfo sk_info() {
    KernelInfo k;
    k.func = reinterpret_cast<const void *>(splitk_gemm_kernel<C>);
    k.threads = C::THREADS;
    k.smem_bytes = C::SMEM_BYTES;
    k.stages = C::STAGES;
    k.block_m = C::NM;
    k.block_n = 128;
    k.block_k = C::BK;
    return k;
}

template <class C>
cudaError_t launch_sg(const SgLaunch &L) {
    auto kern = splitk_grid_kernel<C>;
    static int attr_done[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_done[dev] = 1;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(L.p.grid, 1, 1);
    cfg.blockDim = dim3(C::THREADS, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = L.stream;
    cudaLaunchAttribute attr[1];
    int na = 0;
    if (L.pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = na ? attr : nullptr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, kern, L.tmW, L.tmX, L.p);
}

template <class C>
KernelInfo sg_info() {
    KernelInfo k;
    k.func = reinterpret_cast<const void *>(splitk_grid_kernel<C>);
    k.threads = C::THREADS;
    k.smem_bytes = C::SMEM_BYTES;
    k.stages = C::STAGES;
    k.block_m = C::NM;
    k.block_n = 128;
    k.block_k = C::BK;
    return k;
}

// Instantiate and look up every (epilogue, axis, layout, tile) combination of
// one dtype.  NONE ignores the bias, so it exists for the ROW axis only.
#define GEMM_EPI_TC_FIND(NAME, DTV)                                                                     \
    template <int CG, int EPI, int AXIS, bool BMN, int BN>                                              \
    static bool NAME##_leaf(TcLauncher *l, KernelInfo *i) {                                             \
        constexpr int ES = (DTV) == DT_E4M3 ? 1 : 2;                                                    \
        constexpr int STG = tc_stages(tc_katoms(128 * 128 + (BN / CG) * 128) * (128 * 128 + (BN / CG) * 128));                                     \
        if constexpr (BMN && (BN / CG) % (128 / ES) != 0) {                                             \
            return false; /* an MN-major B half-tile narrower than one 128-byte box */                  \
        } else if constexpr (BN == 512 && (CG != 2 || EPI == EPI_DRELU)) {                              \
            return false; /* 512-wide tiles: CTA pairs, forward epilogues */                            \
        } else {                                                                                        \
            using C = TcCfg<DTV, EPI, AXIS, BMN, BN, CG, STG>;                                          \
            *l = &launch_tc<C>;                                                                         \
            *i = tc_info<C>();                                                                          \
            return true;                                                                                \
        }                                                                                               \
    }                                                                                                   \
    template <int CG, int EPI, int AXIS, bool BMN>                                                      \
    static bool NAME##_bn(int bn, TcLauncher *l, KernelInfo *i) {                                       \
        if (bn == 512) return NAME##_leaf<CG, EPI, AXIS, BMN, 512>(l, i);                               \
        if (bn == 256) return NAME##_leaf<CG, EPI, AXIS, BMN, 256>(l, i);                               \
        if (bn == 128) return NAME##_leaf<CG, EPI, AXIS, BMN, 128>(l, i);                               \
        return false;                                                                                   \
    }                                                                                                   \
    template <int CG, int EPI, int AXIS>                                                                \
    static bool NAME##_mn(bool bmn, int bn, TcLauncher *l, KernelInfo *i) {                             \
        return bmn ? NAME##_bn<CG, EPI, AXIS, true>(bn, l, i) : NAME##_bn<CG, EPI, AXIS, false>(bn, l, i); \
    }                                                                                                   \
    template <int CG>                                                                                   \
    static bool NAME##_cg(int epi, int axis, bool bmn, int bn, TcLauncher *l, KernelInfo *i) {          \
        switch (epi) {                                                                                  \
        case EPI_NONE: return NAME##_mn<CG, EPI_NONE, AXIS_ROW>(bmn, bn, l, i);                         \
        case EPI_BIAS: return axis ? NAME##_mn<CG, EPI_BIAS, AXIS_COL>(bmn, bn, l, i)                   \
                                   : NAME##_mn<CG, EPI_BIAS, AXIS_ROW>(bmn, bn, l, i);                  \
        case EPI_RELU: return axis ? NAME##_mn<CG, EPI_RELU, AXIS_COL>(bmn, bn, l, i)                   \
                                   : NAME##_mn<CG, EPI_RELU, AXIS_ROW>(bmn, bn, l, i);                  \
        case EPI_RELU_AUX: return axis ? NAME##_mn<CG, EPI_RELU_AUX, AXIS_COL>(bmn, bn, l, i)           \
                                       : NAME##_mn<CG, EPI_RELU_AUX, AXIS_ROW>(bmn, bn, l, i);          \
        case EPI_GELU: return axis ? NAME##_mn<CG, EPI_GELU, AXIS_COL>(bmn, bn, l, i)                   \
                                   : NAME##_mn<CG, EPI_GELU, AXIS_ROW>(bmn, bn, l, i);                  \
        case EPI_TANH: return axis ? NAME##_mn<CG, EPI_TANH, AXIS_COL>(bmn, bn, l, i)                   \
                                   : NAME##_mn<CG, EPI_TANH, AXIS_ROW>(bmn, bn, l, i);                  \
        case EPI_DRELU: return axis ? NAME##_mn<CG, EPI_DRELU, AXIS_COL>(bmn, bn, l, i)                 \
                                    : NAME##_mn<CG, EPI_DRELU, AXIS_ROW>(bmn, bn, l, i);                \
        }                                                                                               \
        return false;                                                                                   \
    }                                                                                                   \
    bool NAME(int cg, int epi, int axis, bool bmn, int bn, TcLauncher *l, KernelInfo *i) {              \
        if (cg == 1) return NAME##_cg<1>(epi, axis, bmn, bn, l, i);                                     \
        if (cg == 2) return NAME##_cg<2>(epi, axis, bmn, bn, l, i);                                     \
        return false;                                                                                   \
    }

#define GEMM_EPI_SK_FIND(NAME, DTV)                                                                     \
    template <int EPI, int AXIS, bool WMN, int NM>                                                      \
    static bool NAME##_leaf(SkLauncher *l, KernelInfo *i) {                                             \
        using C = SkCfg<DTV, EPI, AXIS, WMN, NM, sk_stages(NM)>;                                        \
        *l = &launch_sk<C>;                                                                             \
        *i = sk_info<C>();                                                                              \
        return true;                                                                                    \
    }                                                                                                   \
    template <int EPI, int AXIS, bool WMN>                                                              \
    static bool NAME##_nm(int nm, SkLauncher *l, KernelInfo *i) {                                       \
        switch (nm) {                                                                                   \
        case 16: return NAME##_leaf<EPI, AXIS, WMN, 16>(l, i);                                          \
        case 32: return NAME##_leaf<EPI, AXIS, WMN, 32>(l, i);                                          \
        case 64: return NAME##_leaf<EPI, AXIS, WMN, 64>(l, i);                                          \
        case 128: return NAME##_leaf<EPI, AXIS, WMN, 128>(l, i);                                        \
        }                                                                                               \
        return false;                                                                                   \
    }                                                                                                   \
    template <int EPI, int AXIS>                                                                        \
    static bool NAME##_mn(bool wmn, int nm, SkLauncher *l, KernelInfo *i) {                             \
        return wmn ? NAME##_nm<EPI, AXIS, true>(nm, l, i) : NAME##_nm<EPI, AXIS, false>(nm, l, i);      \
    }                                                                                                   \
    bool NAME(int epi, int axis, bool wmn, int nm, SkLauncher *l, KernelInfo *i) {                      \
        switch (epi) {                                                                                  \
        case EPI_NONE: return NAME##_mn<EPI_NONE, AXIS_ROW>(wmn, nm, l, i);                             \
        case EPI_BIAS: return axis ? NAME##_mn<EPI_BIAS, AXIS_COL>(wmn, nm, l, i)                       \
                                   : NAME##_mn<EPI_BIAS, AXIS_ROW>(wmn, nm, l, i);                      \
        case EPI_RELU: return axis ? NAME##_mn<EPI_RELU, AXIS_COL>(wmn, nm, l, i)                       \
                                   : NAME##_mn<EPI_RELU, AXIS_ROW>(wmn, nm, l, i);                      \
        case EPI_RELU_AUX: return axis ? NAME##_mn<EPI_RELU_AUX, AXIS_COL>(wmn, nm, l, i)               \
                                       : NAME##_mn<EPI_RELU_AUX, AXIS_ROW>(wmn, nm, l, i);              \
        case EPI_GELU: return axis ? NAME##_mn<EPI_GELU, AXIS_COL>(wmn, nm, l, i)                       \
                                   : NAME##_mn<EPI_GELU, AXIS_ROW>(wmn, nm, l, i);                      \
        case EPI_TANH: return axis ? NAME##_mn<EPI_TANH, AXIS_COL>(wmn, nm, l, i)                       \
                                   : NAME##_mn<EPI_TANH, AXIS_ROW>(wmn, nm, l, i);                      \
        }                                                                                               \
        return false;                                                                                   \
    }

#define GEMM_EPI_SG_FIND(NAME, DTV)                                                                     \
    template <int EPI, int AXIS, bool WMN, int NM>                                                      \
    static bool NAME##_leaf(SgLauncher *l, KernelInfo *i) {                                             \
        using C = SgCfg<DTV, EPI, AXIS, WMN, NM, sg_stages(NM)>;                                        \
        *l = &launch_sg<C>;                                                                             \
        *i = sg_info<C>();                                                                              \
        return true;                                                                                    \
    }                                                                                                   \
    template <int EPI, int AXIS, bool WMN>                                                              \
    static bool NAME##_nm(int nm, SgLauncher *l, KernelInfo *i) {                                       \
        switch (nm) {                                                                                   \
        case 16: return NAME##_leaf<EPI, AXIS, WMN, 16>(l, i);                                          \
        case 32: return NAME##_leaf<EPI, AXIS, WMN, 32>(l, i);                                          \
        case 64: return NAME##_leaf<EPI, AXIS, WMN, 64>(l, i);                                          \
        case 128: return NAME##_leaf<EPI, AXIS, WMN, 128>(l, i);                                        \
        }                                                                                               \
        return false;                                                                                   \
    }                                                                                                   \
    template <int EPI, int AXIS>                                                                        \
    static bool NAME##_mn(bool wmn, int nm, SgLauncher *l, KernelInfo *i) {                             \
        return wmn ? NAME##_nm<EPI, AXIS, true>(nm, l, i) : NAME##_nm<EPI, AXIS, false>(nm, l, i);      \
    }                                                                                                   \
    bool NAME(int epi, int axis, bool wmn, int nm, SgLauncher *l, KernelInfo *i) {                      \
        switch (epi) {                                                                                  \
        case EPI_NONE: return NAME##_mn<EPI_NONE, AXIS_ROW>(wmn, nm, l, i);                             \
        case EPI_BIAS: return axis ? NAME##_mn<EPI_BIAS, AXIS_COL>(wmn, nm, l, i)                       \
                                   : NAME##_mn<EPI_BIAS, AXIS_ROW>(wmn, nm, l, i);                      \
        case EPI_RELU: return axis ? NAME##_mn<EPI_RELU, AXIS_COL>(wmn, nm, l, i)                       \
                                   : NAME##_mn<EPI_RELU, AXIS_ROW>(wmn, nm, l, i);                      \
        case EPI_RELU_AUX: return axis ? NAME##_mn<EPI_RELU_AUX, AXIS_COL>(wmn, nm, l, i)               \
                                       : NAME##_mn<EPI_RELU_AUX, AXIS_ROW>(wmn, nm, l, i);              \
        case EPI_GELU: return axis ? NAME##_mn<EPI_GELU, AXIS_COL>(wmn, nm, l, i)                       \
                                   : NAME##_mn<EPI_GELU, AXIS_ROW>(wmn, nm, l, i);                      \
        case EPI_TANH: return axis ? NAME##_mn<EPI_TANH, AXIS_COL>(wmn, nm, l, i)                       \
                                   : NAME##_mn<EPI_TANH, AXIS_ROW>(wmn, nm, l, i);                      \
        }                                                                                               \
        return false;                                                                                   \
    }

}  // namespace gemm_epi
