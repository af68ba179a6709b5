// Gather and fused kernels instantiated for the LdF32x1 row loader.
#include "kernels.cuh"

namespace dlrm {
DLRM_INSTANTIATE_LOADER(LdF32x1, f32x1)
}  // namespace dlrm
