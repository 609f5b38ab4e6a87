// Instantiations of the unfused bias/activation kernel (the stepwise baseline).
#include "bias_act.cuh"
#include "kernels.h"

namespace gemm_epi {

template <int DT, int EPI, int AXIS>
static cudaError_t launch_ba(void *D, const void *bias, uint32_t *aux, int m, int n, int64_t pitch_words,
                             int grid, cudaStream_t stream) {
    const int64_t total = (int64_t)m * pitch_words;
    if (total == 0) return cudaSuccess;
    bias_act_kernel<DT, EPI, AXIS><<<grid, 256, 0, stream>>>(D, bias, aux, m, n, pitch_words, total);
    return cudaGetLastError();
}

template <int DT, int EPI>
static BiasActLauncher pick_axis(int axis) {
    return axis ? &launch_ba<DT, EPI, AXIS_COL> : &launch_ba<DT, EPI, AXIS_ROW>;
}

template <int DT>
static BiasActLauncher pick_epi(int epi, int axis) {
    switch (epi) {
    case EPI_BIAS: return pick_axis<DT, EPI_BIAS>(axis);
    case EPI_RELU: return pick_axis<DT, EPI_RELU>(axis);
    case EPI_RELU_AUX: return pick_axis<DT, EPI_RELU_AUX>(axis);
    case EPI_GELU: return pick_axis<DT, EPI_GELU>(axis);
    case EPI_TANH: return pick_axis<DT, EPI_TANH>(axis);
    case EPI_DRELU: return &launch_ba<DT, EPI_DRELU, AXIS_ROW>;   // no bias: the axis plays no part
    }
    return nullptr;
}

bool find_bias_act(int dt, int epi, int axis, BiasActLauncher *launch) {
    BiasActLauncher l = nullptr;
    switch (dt) {
    case DT_F16: l = pick_epi<DT_F16>(epi, axis); break;
    case DT_BF16: l = pick_epi<DT_BF16>(epi, axis); break;
    case DT_E4M3: l = pick_epi<DT_E4M3>(epi, axis); break;
    }
    *launch = l;
    return l != nullptr;
}

}  // namespace gemm_epi
