// Internal launchers of the stage's kernels (host side, not part of the C ABI).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "device_common.cuh"

namespace dlrm {

// Blocks of the fused kernel that the register allocation keeps resident per SM.
#ifndef DLRM_FUSED_MIN_BLOCKS
#define DLRM_FUSED_MIN_BLOCKS 8
#endif

// Which row loader a launch uses.
enum LoaderKind { kLdF32x4 = 0, kLdF32x1 = 1, kLdBF16x8 = 2, kLdBF16x1 = 3, kLdF32x4S = 4 };

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

// cuTensorMapEncodeTiled, looked up once through the runtime's driver entry
// point (null if the driver does not provide it); the MLP layers' TMA loads
// use it.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled();

// Records a failed CUDA call for dlrm_last_cuda_error() and returns DLRM_ERR_CUDA.
int cuda_fail(cudaError_t e);

// One pair of launchers per loader (inst_*.cu).
cudaError_t launch_gather_f32x4(const GatherLaunch& a);
cudaError_t launch_gather_f32x4s(const GatherLaunch& a);
cudaError_t launch_gather_f32x1(const GatherLaunch& a);
cudaError_t launch_gather_bf16x8(const GatherLaunch& a);
cudaError_t launch_gather_bf16x1(const GatherLaunch& a);
cudaError_t launch_fused_f32x4(const FusedLaunch& a);
cudaError_t launch_fused_f32x4s(const FusedLaunch& a);
cudaError_t launch_fused_f32x1(const FusedLaunch& a);
cudaError_t launch_fused_bf16x8(const FusedLaunch& a);
cudaError_t launch_fused_bf16x1(const FusedLaunch& a);

// Shared-memory bytes that one sample's features take in the dot phase.
int64_t interact_smem_per_sample(int F, int D);

// Everything a gather launch needs besides its outputs.
struct GatherPlan {
  const TableParams* tp;
  BagParams bp;
  int B, F, D;
  int pool;    // PoolKind
  int loader;  // LoaderKind
  int esz;     // table element bytes (4 or 2)
};

// Process-wide choice of gather path (dlrm_set_gather_path).
int gather_path();
void set_gather_path(int path);
// The path (DLRM_PATH_LDG) of this thread's last gather launch.
int last_path();

// Picks the shape, then launches.
cudaError_t launch_embbag(const GatherPlan& g, float* out, cudaStream_t stream);

cudaError_t launch_fused(const GatherPlan& g, const float* dense, float* pooled_out,
                         float* inter_out, int concat_dense, int64_t smem_limit,
                         cudaStream_t stream);

cudaError_t launch_interact(const float* dense, const float* emb, int B, int F, int D, float* out,
                            bool vec_ok, int64_t smem_limit, cudaStream_t stream);

cudaError_t launch_pair_decode(int64_t p0, int64_t count, int32_t* i_out, int32_t* j_out,
                               cudaStream_t stream);

int64_t launch_count();

cudaError_t launch_probe_wait(int64_t limit, int32_t* status, cudaStream_t stream);
cudaError_t launch_probe_row_gather(const void* table, int64_t rows, int chunks, int64_t count,
                                    uint64_t seed, uint32_t* sink, cudaStream_t stream);
// Counts one kernel launch of this library (dlrm_launch_count).
void note_launch();

}  // namespace dlrm
