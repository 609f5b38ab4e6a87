// Instantiations of the small-m split-K kernel for f16 operands.
#include "kernels.h"
namespace gemm_epi {
GEMM_EPI_SK_FIND(find_sk_f16, DT_F16)
}  // namespace gemm_epi
