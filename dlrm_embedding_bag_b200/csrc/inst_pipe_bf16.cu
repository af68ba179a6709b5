// Pipelined register-load kernels instantiated for bf16 tables (128-bit loads).
#include <algorithm>

#include "pipe_kernels.cuh"

namespace dlrm {
cudaError_t launch_pipe_gather_bf16(const PipeLaunch& a) {
  DLRM_PIPE_DISPATCH(run_pipe_gather, LdBF16x8, a);
}
cudaError_t launch_pipe_fused_bf16(const PipeLaunch& a) {
  DLRM_PIPE_DISPATCH(run_pipe_fused, LdBF16x8, a);
}
}  // namespace dlrm
