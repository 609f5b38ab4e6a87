// Instantiations of the grid-wide small-m split-K kernel for bf16 operands.
#include "kernels.h"
namespace gemm_epi {
GEMM_EPI_SG_FIND(find_sg_bf16, DT_BF16)
}  // namespace gemm_epi
