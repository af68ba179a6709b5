// TMA gather-path kernels instantiated for bf16 tables.
#include <algorithm>

#include "tma_kernels.cuh"

namespace dlrm {
cudaError_t launch_tma_gather_bf16(const TmaLaunch& a) { DLRM_TMA_DISPATCH(run_tma_gather, 2, a); }
cudaError_t launch_tma_fused_bf16(const TmaLaunch& a) { DLRM_TMA_DISPATCH(run_tma_fused, 2, a); }
}  // namespace dlrm
