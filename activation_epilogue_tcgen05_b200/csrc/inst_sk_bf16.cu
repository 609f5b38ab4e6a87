// Instantiations of the small-m split-K kernel for bf16 operands.
#include "kernels.h"
namespace gemm_epi {
GEMM_EPI_SK_FIND(find_sk_bf16, DT_BF16)
}  // namespace gemm_epi
