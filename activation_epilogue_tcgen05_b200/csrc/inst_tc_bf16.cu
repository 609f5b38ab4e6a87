// Instantiations of the persistent tcgen05 kernel for bf16 operands.
#include "kernels.h"
namespace gemm_epi {
GEMM_EPI_TC_FIND(find_tc_bf16, DT_BF16)
}  // namespace gemm_epi
