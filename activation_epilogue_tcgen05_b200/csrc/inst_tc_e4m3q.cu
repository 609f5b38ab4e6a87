// Instantiations of the persistent tcgen05 kernel for e4m3 operands with an e4m3
// output quantised in the epilogue (the MLP block's intermediate).  Epilogues:
// NONE (ROW), BIAS, RELU and GELU, either bias axis.
#include "kernels.h"

namespace gemm_epi {

template <int CG, int EPI, int AXIS, bool BMN, int BN>
static bool q_leaf(TcLauncher *l, KernelInfo *i) {
    constexpr int STG = tc_stages(tc_katoms(128 * 128 + (BN / CG) * 128) * (128 * 128 + (BN / CG) * 128));
    if constexpr (BMN && (BN / CG) % 128 != 0) {
        return false;   // an MN-major B half-tile narrower than one 128-byte box
    } else {
        using C = TcCfg<DT_E4M3, EPI, AXIS, BMN, BN, CG, STG, true>;
        *l = &launch_tc<C>;
        *i = tc_info<C>();
        return true;
    }
}

template <int CG, int EPI, int AXIS, bool BMN>
static bool q_bn(int bn, TcLauncher *l, KernelInfo *i) {
    if (bn == 256) return q_leaf<CG, EPI, AXIS, BMN, 256>(l, i);
    if (bn == 128) return q_leaf<CG, EPI, AXIS, BMN, 128>(l, i);
    return false;
}

template <int CG, int EPI, int AXIS>
static bool q_mn(bool bmn, int bn, TcLauncher *l, KernelInfo *i) {
    return bmn ? q_bn<CG, EPI, AXIS, true>(bn, l, i) : q_bn<CG, EPI, AXIS, false>(bn, l, i);
}

template <int CG>
static bool q_cg(int epi, int axis, bool bmn, int bn, TcLauncher *l, KernelInfo *i) {
    switch (epi) {
    case EPI_NONE: return q_mn<CG, EPI_NONE, AXIS_ROW>(bmn, bn, l, i);
    case EPI_BIAS: return axis ? q_mn<CG, EPI_BIAS, AXIS_COL>(bmn, bn, l, i) : q_mn<CG, EPI_BIAS, AXIS_ROW>(bmn, bn, l, i);
    case EPI_RELU: return axis ? q_mn<CG, EPI_RELU, AXIS_COL>(bmn, bn, l, i) : q_mn<CG, EPI_RELU, AXIS_ROW>(bmn, bn, l, i);
    case EPI_GELU: return axis ? q_mn<CG, EPI_GELU, AXIS_COL>(bmn, bn, l, i) : q_mn<CG, EPI_GELU, AXIS_ROW>(bmn, bn, l, i);
    }
    return false;
}

bool find_tc_e4m3_q(int cg, int epi, int axis, bool bmn, int bn, TcLauncher *l, KernelInfo *i) {
    if (cg == 1) return q_cg<1>(epi, axis, bmn, bn, l, i);
    if (cg == 2) return q_cg<2>(epi, axis, bmn, bn, l, i);
    return false;
}

}  // namespace gemm_epi
