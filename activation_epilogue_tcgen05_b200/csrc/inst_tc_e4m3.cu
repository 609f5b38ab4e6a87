// Instantiations of the persistent tcgen05 kernel for e4m3 operands.
#include "kernels.h"
namespace gemm_epi {
GEMM_EPI_TC_FIND(find_tc_e4m3, DT_E4M3)
}  // namespace gemm_epi
