// Instantiations of the small-m split-K kernel for e4m3 operands with an e4m3 output
// quantised in the epilogue.
#include "kernels.h"
namespace gemm_epi {
bool find_sk_e4m3_q(int epi, int axis, bool w_mn, int nm, SkLauncher *l, KernelInfo *i) {
    return SkFindQ::find(epi, axis, w_mn, nm, l, i);
}
}  // namespace gemm_epi
