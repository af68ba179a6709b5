// Gather and fused kernels instantiated for the LdBF16x8 row loader.
#include "kernels.cuh"

namespace dlrm {
DLRM_INSTANTIATE_LOADER(LdBF16x8, bf16x8)
}  // namespace dlrm
