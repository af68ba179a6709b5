// Pipelined register-load kernels instantiated for f32 tables (128-bit loads).
#include <algorithm>

#include "pipe_kernels.cuh"

namespace dlrm {
cudaError_t launch_pipe_gather_f32(const PipeLaunch& a) {
  DLRM_PIPE_DISPATCH(run_pipe_gather, LdF32x4, a);
}
cudaError_t launch_pipe_fused_f32(const PipeLaunch& a) {
  DLRM_PIPE_DISPATCH(run_pipe_fused, LdF32x4, a);
}
}  // namespace dlrm
