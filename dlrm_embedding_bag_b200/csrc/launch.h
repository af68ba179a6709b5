// Internal launchers of the stage's kernels (host side, not part of the C ABI).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "device_common.cuh"

namespace dlrm {

// Blocks of the fused kernel that the register allocation keeps resident per SM.
#ifndef DLRM_FUSED_MIN_BLOCKS
#define DLRM_FUSED_MIN_BLOCKS 4
#endif

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

// cuTensorMapEncodeTiled, looked up once through the runtime's driver entry
// point (null if the driver does not provide it).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled();

// Records a failed CUDA call for dlrm_last_cuda_error() and returns DLRM_ERR_CUDA.
int cuda_fail(cudaError_t e);

// Tensor maps of the TMA gather path: one 2-D map per table ({D, rows},
// box {D, 1}), passed by value in the kernel's parameter block.
constexpr int kTmaMaxTables = 64;
struct alignas(64) TmaParams {
  CUtensorMap map[kTmaMaxTables];
  int32_t rows[kTmaMaxTables];
};

struct TmaLaunch {
  const TmaParams* tp;
  BagParams bp;
  int B, F, D;
  int G;     // lanes per unit (8 or 16)
  int cpl;   // 16-byte row chunks per lane (1 or 2)
  int pool;  // PoolKind
  float* out;  // gather-only output
  // fused
  const float* dense;
  float* pooled_out;
  float* inter_out;
  int concat_dense;
  int S, lq;
  int64_t smem_limit;
  int sms;
  cudaStream_t stream;
};

// The persistent pipelined register-load path.
struct PipeLaunch {
  const TableParams* tp;
  BagParams bp;
  int B, F, D;
  int G, cpl;  // lanes per unit, 16-byte chunks per lane
  int pool;
  float* out;  // gather-only output
  const float* dense;
  float* pooled_out;
  float* inter_out;
  int concat_dense;
  int S, lq;
  int64_t smem;
  int sms;
  cudaStream_t stream;
};

cudaError_t launch_pipe_gather_f32(const PipeLaunch& a);
cudaError_t launch_pipe_gather_bf16(const PipeLaunch& a);
cudaError_t launch_pipe_fused_f32(const PipeLaunch& a);
cudaError_t launch_pipe_fused_bf16(const PipeLaunch& a);

cudaError_t launch_tma_gather_f32(const TmaLaunch& a);
cudaError_t launch_tma_gather_bf16(const TmaLaunch& a);
cudaError_t launch_tma_fused_f32(const TmaLaunch& a);
cudaError_t launch_tma_fused_bf16(const TmaLaunch& a);

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

// Everything a gather launch needs besides its outputs.
struct GatherPlan {
  const TableParams* tp;
  BagParams bp;
  int B, F, D;
  int pool;             // PoolKind
  int loader;           // LoaderKind of the register (LDG) path
  int esz;              // table element bytes (4 or 2)
  bool tma_ok;          // tables and shape qualify for the TMA gather path
  const int64_t* rows;  // host row counts, or null (then the maps span INT32_MAX rows)
};

// Process-wide choice of gather path (dlrm_set_gather_path).
int gather_path();
void set_gather_path(int path);
// The path (DLRM_PATH_LDG / DLRM_PATH_TMA) of this thread's last gather launch.
int last_path();

// Picks the path and shape, then launches.
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
// Counts one kernel launch of this library (dlrm_launch_count).
void note_launch();

}  // namespace dlrm
