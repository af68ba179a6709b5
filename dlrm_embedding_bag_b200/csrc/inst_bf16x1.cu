// Gather and fused kernels instantiated for the LdBF16x1 row loader.
#include "kernels.cuh"

namespace dlrm {
DLRM_INSTANTIATE_LOADER(LdBF16x1, bf16x1)
}  // namespace dlrm
