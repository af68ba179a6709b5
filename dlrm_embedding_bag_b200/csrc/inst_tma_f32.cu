// TMA gather-path kernels instantiated for f32 tables.
#include <algorithm>

#include "tma_kernels.cuh"

namespace dlrm {
cudaError_t launch_tma_gather_f32(const TmaLaunch& a) { DLRM_TMA_DISPATCH(run_tma_gather, 4, a); }
cudaError_t launch_tma_fused_f32(const TmaLaunch& a) { DLRM_TMA_DISPATCH(run_tma_fused, 4, a); }
}  // namespace dlrm
