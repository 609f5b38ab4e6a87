// find_at.cuh -- lookup of the persistent-kernel instantiations with A stored (k, m);
// included only by the inst_tc_*_at.cu units that instantiate them.
#pragma once
#include "kernels.h"

namespace gemm_epi {

// A stored (k, m): the forward epilogues, both bias axes and B layouts, 256-wide tiles only.
template <int DTV>
struct TcFindAT {
    template <int CG, int EPI, int AXIS, bool BMN>
    static bool leaf(TcLauncher *l, KernelInfo *i) {
        constexpr int ES = DTV == DT_E4M3 ? 1 : 2;
        constexpr int STG = tc_stages(tc_katoms(128 * 128 + (256 / CG) * 128) * (128 * 128 + (256 / CG) * 128));
        if constexpr (BMN && (256 / CG) % (128 / ES) != 0) {
            return false;
        } else {
            using C = TcCfg<DTV, EPI, AXIS, BMN, 256, CG, STG, false, true>;
            *l = &launch_tc<C>;
            *i = tc_info<C>();
            return true;
        }
    }
    template <int CG, int EPI, int AXIS>
    static bool mn(bool bmn, TcLauncher *l, KernelInfo *i) {
        return bmn ? leaf<CG, EPI, AXIS, true>(l, i) : leaf<CG, EPI, AXIS, false>(l, i);
    }
    template <int CG, int EPI>
    static bool ax(int axis, bool bmn, TcLauncher *l, KernelInfo *i) {
        return axis ? mn<CG, EPI, AXIS_COL>(bmn, l, i) : mn<CG, EPI, AXIS_ROW>(bmn, l, i);
    }
    template <int CG>
    static bool epi(int e, int axis, bool bmn, TcLauncher *l, KernelInfo *i) {
        switch (e) {
        case EPI_NONE: return mn<CG, EPI_NONE, AXIS_ROW>(bmn, l, i);
        case EPI_BIAS: return ax<CG, EPI_BIAS>(axis, bmn, l, i);
        case EPI_RELU: return ax<CG, EPI_RELU>(axis, bmn, l, i);
        case EPI_RELU_AUX: return ax<CG, EPI_RELU_AUX>(axis, bmn, l, i);
        case EPI_GELU: return ax<CG, EPI_GELU>(axis, bmn, l, i);
        case EPI_TANH: return ax<CG, EPI_TANH>(axis, bmn, l, i);
        }
        return false;
    }
    static bool find(int cg, int e, int axis, bool bmn, int bn, TcLauncher *l, KernelInfo *i) {
        if (bn != 256) return false;
        if (cg == 1) return epi<1>(e, axis, bmn, l, i);
        if (cg == 2) return epi<2>(e, axis, bmn, l, i);
        return false;
    }
};

}  // namespace gemm_epi
