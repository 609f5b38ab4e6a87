// Instantiations of the persistent tcgen05 kernel for f16 operands with A stored (k, m).
#include "find_at.cuh"
namespace gemm_epi {
bool find_tc_f16_at(int cg, int epi, int axis, bool bmn, int bn, TcLauncher *l, KernelInfo *i) {
    return TcFindAT<DT_F16>::find(cg, epi, axis, bmn, bn, l, i);
}
}  // namespace gemm_epi
