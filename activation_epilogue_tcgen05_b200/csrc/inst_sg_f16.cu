// Instantiations of the grid-wide small-m split-K kernel for f16 operands.
#include "kernels.h"
namespace gemm_epi {
GEMM_EPI_SG_FIND(find_sg_f16, DT_F16)
}  // namespace gemm_epi
