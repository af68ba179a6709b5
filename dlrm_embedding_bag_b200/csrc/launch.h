// Internal launchers of the stage's kernels (host side, not part of the C ABI).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "device_common.cuh"

namespace dlrm {

// Template shape of the gather for a row length D: VEC floats per load, G
// lanes per bag, CPL column chunks per lane, U rows fetched per batch, and the
// number of column windows that cover D.
struct GatherShape {
  int vec, G, cpl, u, ncolwin;
};
GatherShape choose_gather_shape(int D, bool vec_ok);

// Shared-memory bytes that one sample's features take in the dot phase.
int64_t interact_smem_per_sample(int F, int D);

cudaError_t launch_embbag(const TableParams& tp, const int32_t* indices, const int32_t* offsets,
                          int B, int F, int L, int D, float* out, int32_t* status, bool check,
                          bool vec_ok, cudaStream_t stream);

cudaError_t launch_interact(const float* dense, const float* emb, int B, int F, int D, float* out,
                            bool vec_ok, int64_t smem_limit, cudaStream_t stream);

cudaError_t launch_fused(const TableParams& tp, const int32_t* indices, const int32_t* offsets,
                         const float* dense, int B, int F, int L, int D, float* pooled_out,
                         float* inter_out, int concat_dense, int32_t* status, bool check,
                         bool vec_ok, int64_t smem_limit, cudaStream_t stream);

cudaError_t launch_pair_decode(int64_t p0, int64_t count, int32_t* i_out, int32_t* j_out,
                               cudaStream_t stream);

int64_t launch_count();

}  // namespace dlrm
