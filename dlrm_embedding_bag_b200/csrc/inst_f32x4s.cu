// Gather and fused kernels instantiated for the LdF32x4S row loader.
#include "kernels.cuh"

namespace dlrm {
DLRM_INSTANTIATE_LOADER(LdF32x4S, f32x4s)
}  // namespace dlrm
