// Internal launchers of the stage's kernels (host side, not part of the C ABI).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "device_common.cuh"

namespace dlrm {

// Which row loader a launch uses.
enum LoaderKind { kLdF32x4 = 0, kLdF32x1 = 1, kLdBF16x8 = 2, kLdBF16x1 = 3 };

// Template shape of the gather for a row length D: the loader, G lanes per bag,
// CPL column chunks per lane, and the number of column windows that cover D.
struct GatherShape {
  int loader, vec, G, cpl, ncolwin;
};
GatherShape choose_gather_shape(int D, int loader);

struct GatherLaunch {
  const TableParams* tp;
  BagParams bp;
  int B, F, D;
  float* out;
  int pool;  // PoolKind
  GatherShape shape;
  cudaStream_t stream;
};

struct FusedLaunch {
  GatherLaunch g;
  const float* dense;
  float* pooled_out;
  float* inter_out;
  int concat_dense;
  int S, lq;
  int64_t smem;
};

// One pair of launchers per loader (inst_*.cu).
cudaError_t launch_gather_f32x4(const GatherLaunch& a);
cudaError_t launch_gather_f32x1(const GatherLaunch& a);
cudaError_t launch_gather_bf16x8(const GatherLaunch& a);
cudaError_t launch_gather_bf16x1(const GatherLaunch& a);
cudaError_t launch_fused_f32x4(const FusedLaunch& a);
cudaError_t launch_fused_f32x1(const FusedLaunch& a);
cudaError_t launch_fused_bf16x8(const FusedLaunch& a);
cudaError_t launch_fused_bf16x1(const FusedLaunch& a);

// Shared-memory bytes that one sample's features take in the dot phase.
int64_t interact_smem_per_sample(int F, int D);

// Picks the shape and launches; `loader` from the table dtype and alignment.
cudaError_t launch_embbag(const TableParams& tp, const BagParams& bp, int B, int F, int D,
                          float* out, int pool, int loader, cudaStream_t stream);

cudaError_t launch_fused(const TableParams& tp, const BagParams& bp, const float* dense, int B,
                         int F, int D, float* pooled_out, float* inter_out, int concat_dense,
                         int pool, int loader, int64_t smem_limit, cudaStream_t stream);

cudaError_t launch_interact(const float* dense, const float* emb, int B, int F, int D, float* out,
                            bool vec_ok, int64_t smem_limit, cudaStream_t stream);

cudaError_t launch_pair_decode(int64_t p0, int64_t count, int32_t* i_out, int32_t* j_out,
                               cudaStream_t stream);

int64_t launch_count();

}  // namespace dlrm
