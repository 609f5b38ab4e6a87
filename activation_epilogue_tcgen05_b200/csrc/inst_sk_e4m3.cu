// Instantiations of the small-m split-K kernel for e4m3 operands.
#include "kernels.h"
namespace gemm_epi {
GEMM_EPI_SK_FIND(find_sk_e4m3, DT_E4M3)
}  // namespace gemm_epi
