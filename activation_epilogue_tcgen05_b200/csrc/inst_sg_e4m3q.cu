// Instantiations of the grid-wide small-m split-K kernel for e4m3 operands with an e4m3 output
// quantised in the epilogue.
#include "kernels.h"
namespace gemm_epi {

// Grid-wide split-K kernels for e4m3 operands with an e4m3 output quantised in the epilogue:
// NONE (ROW), BIAS, RELU, GELU, either bias axis, every batch width.
struct SgFindQ {
    template <int EPI, int AXIS, bool WMN, int NM>
    static bool leaf(SgLauncher *l, KernelInfo *i) {
        using C = SgCfg<DT_E4M3, EPI, AXIS, WMN, NM, sg_stages(NM), true>;
        *l = &launch_sg<C>;
        *i = sg_info<C>();
        return true;
    }
    template <int EPI, int AXIS, bool WMN>
    static bool nm(int v, SgLauncher *l, KernelInfo *i) {
        switch (v) {
        case 16: return leaf<EPI, AXIS, WMN, 16>(l, i);
        case 32: return leaf<EPI, AXIS, WMN, 32>(l, i);
        case 64: return leaf<EPI, AXIS, WMN, 64>(l, i);
        case 128: return leaf<EPI, AXIS, WMN, 128>(l, i);
        }
        return false;
    }
    template <int EPI, int AXIS>
    static bool mn(bool wmn, int v, SgLauncher *l, KernelInfo *i) {
        return wmn ? nm<EPI, AXIS, true>(v, l, i) : nm<EPI, AXIS, false>(v, l, i);
    }
    template <int EPI>
    static bool ax(int axis, bool wmn, int v, SgLauncher *l, KernelInfo *i) {
        return axis ? mn<EPI, AXIS_COL>(wmn, v, l, i) : mn<EPI, AXIS_ROW>(wmn, v, l, i);
    }
    static bool find(int epi, int axis, bool wmn, int v, SgLauncher *l, KernelInfo *i) {
        switch (epi) {
        case EPI_NONE: return mn<EPI_NONE, AXIS_ROW>(wmn, v, l, i);
        case EPI_BIAS: return ax<EPI_BIAS>(axis, wmn, v, l, i);
        case EPI_RELU: return ax<EPI_RELU>(axis, wmn, v, l, i);
        case EPI_GELU: return ax<EPI_GELU>(axis, wmn, v, l, i);
        }
        return false;
    }
};

bool find_sg_e4m3_q(int epi, int axis, bool w_mn, int nm, SgLauncher *l, KernelInfo *i) {
    return SgFindQ::find(epi, axis, w_mn, nm, l, i);
}
}  // namespace gemm_epi
