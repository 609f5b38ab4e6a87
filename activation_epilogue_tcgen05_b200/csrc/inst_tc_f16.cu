// Instantiations of the persistent tcgen05 kernel for f16 operands.
#include "kernels.h"
namespace gemm_epi {
GEMM_EPI_TC_FIND(find_tc_f16, DT_F16)
}  // namespace gemm_epi
