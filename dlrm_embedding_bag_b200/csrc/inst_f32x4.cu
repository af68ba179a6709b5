// Gather and fused kernels instantiated for the LdF32x4 row loader.
#include "kernels.cuh"

namespace dlrm {
DLRM_INSTANTIATE_LOADER(LdF32x4, f32x4)
}  // namespace dlrm
