// Instantiations of the grid-wide small-m split-K kernel for e4m3 operands.
#include "kernels.h"
namespace gemm_epi {
GEMM_EPI_SG_FIND(find_sg_e4m3, DT_E4M3)
}  // namespace gemm_epi
