// DLRMv1 MLP layer on the sm_100a tensor cores: Y = act([A_lo | A_hi] W^T + bias)
// (luminal compare main...vanilla-pytorch, matmul2d.rs: linear_bias,
// linear_bias_relu, linear_bias_sigmoid and the split-A forms), plus the f32 ->
// bf16 conversion that feeds it. Declared in dlrm_mlp.h.
//
// Persistent, warp-specialised kernel: CTA c walks the 128 x BN tiles
// t = c, c + gridDim.x, ... (N tiles fastest, so CTAs running side by side
// share A rows in L2). Ten warps:
//   - warp 0 (one thread) streams 64-wide K blocks of A (128 x 64 bf16) and W
//     (BN x 64) into a 3- or 4-stage shared-memory ring with 2-D TMA loads (128-byte
//     swizzle), running ahead across tiles; K blocks 0..nkb_lo-1 read A_lo,
//     the rest read A_hi, and W's column offset follows, so the
//     concatenation is never built;
//   - warp 1 allocates tensor memory for two f32 accumulators (2 x BN
//     columns) and one thread issues four tcgen05.mma (K = 16 each) per
//     stage into the tile's accumulator, committing each stage back to the
//     producer and each finished accumulator to the epilogue;
//   - warps 2-9 read the finished accumulator (warp w owns TMEM lanes
//     32*(w%4)..+31 and half of the columns), add the bias, apply the
//     activation and store f32 and/or bf16, then hand the accumulator back -
//     so the epilogue of tile i runs while the MMAs of tile i+1 fill the
//     other accumulator.
// Every wait on an mbarrier is bounded; a wait that runs out sets
// DLRM_FLAG_TIMEOUT in the optional status word, ends that role's loop, and
// the CTA still frees its tensor memory and exits.
#include <algorithm>
#include <climits>
#include <cstdint>

#include <cuda_bf16.h>

#include "dlrm_mlp.h"
#include "launch.h"
#include "tcgen05_common.cuh"

namespace dlrm {
namespace {

constexpr int kLinBM = 128;    // rows of a tile (tcgen05 M)
constexpr int kLinBK = 64;     // K per stage: 64 bf16 = one 128-byte swizzle row
// Shared-memory ring depth: 4 stages, except with 256-column tiles (48 KB
// stages) next to the f32 output staging, where only 3 fit.
template <int BN, bool F32S>
constexpr int lin_stages() { return (BN >= 256 && F32S) ? 3 : 4; }
constexpr int kLinEpiWarps = 8;  // two per TMEM lane quarter, each half of the columns
constexpr int kLinThreads = 64 + 32 * kLinEpiWarps;  // producer warp, MMA warp, epilogue
constexpr long long kLinWaitLimit = 200000000LL;  // clock cycles, about 0.1 s

template <int BN, bool F32S>
struct LinSmem {
  static constexpr int kStages = lin_stages<BN, F32S>();
  static constexpr int kA = kLinBM * kLinBK * 2;
  static constexpr int kB = BN * kLinBK * 2;
  static constexpr int kStage = kA + kB;
  // After the ring: each epilogue warp's output staging (a 32 x 32 f32 tile in
  // the 128-byte swizzled layout when F32S -- the f32 output goes out through
  // TMA --, then a 32 x 32 bf16 tile in the 64-byte swizzled layout), its slice
  // of the tile's bias, then the barriers full[S], empty[S], acc_full[2],
  // acc_empty[2] and the TMEM slot.
  static constexpr int kStage32 = F32S ? 32 * 32 * 4 : 0;
  static constexpr int kStage16 = 32 * 32 * 2;
  static constexpr int kStaging = kStages * kStage;
  static constexpr int kBias = kStaging + kLinEpiWarps * (kStage32 + kStage16);
  static constexpr int kBars = kBias + kLinEpiWarps * (BN / 2) * 4;
  static constexpr int kTotal = kBars + (2 * kStages + 4) * 8 + 8 + 1024;  // + alignment
};

struct LinearArgs {
  const float* bias;
  float* y_f32;
  uint16_t* y_bf16;
  int64_t ldy_f32, ldy_bf16;
  int M, N, k_lo, nkb_lo, nkb_hi;
  int tiles_n, tiles;
  int tma_f32, tma_bf16;  // write that output through TMA stores (see the launcher)
  int32_t* status;
};

template <int ACT>
__device__ __forceinline__ float activate(float x) {
  if constexpr (ACT == DLRM_ACT_RELU) {
    return x > 0.f ? x : 0.f;
  } else if constexpr (ACT == DLRM_ACT_SIGMOID) {
    return __fdiv_rn(1.f, __fadd_rn(1.f, expf(-x)));
  } else {
    return x;
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(lo))) |
         (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(hi))) << 16);
}

// Store 32 consecutive results of one row (columns nb .. nb+31, clipped to N).
__device__ __forceinline__ void store_chunk32(const LinearArgs& args, int row, int nb,
                                              const float (&v)[32], bool f32_vec, bool bf_vec) {
  if (row >= args.M) return;
  const bool whole = nb + 32 <= args.N;
  if (args.y_f32 != nullptr) {
    float* y = args.y_f32 + static_cast<int64_t>(row) * args.ldy_f32 + nb;
    if (whole && f32_vec) {
#pragma unroll
      for (int q = 0; q < 8; ++q)
        reinterpret_cast<float4*>(y)[q] =
            make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (nb + j < args.N) y[j] = v[j];
    }
  }
  if (args.y_bf16 != nullptr) {
    uint16_t* y = args.y_bf16 + static_cast<int64_t>(row) * args.ldy_bf16 + nb;
    if (whole && bf_vec) {
#pragma unroll
      for (int q = 0; q < 4; ++q)
        reinterpret_cast<uint4*>(y)[q] = make_uint4(
            pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
            pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (nb + j < args.N) y[j] = __bfloat16_as_ushort(__float2bfloat16_rn(v[j]));
    }
  }
}

template <int BN, int ACT, bool F32S>
__global__ void __launch_bounds__(kLinThreads, 1)
    linear_bf16_kernel(const __grid_constant__ CUtensorMap map_a_lo,
                       const __grid_constant__ CUtensorMap map_a_hi,
                       const __grid_constant__ CUtensorMap map_w,
                       const __grid_constant__ CUtensorMap map_y32,
                       const __grid_constant__ CUtensorMap map_y16, const LinearArgs args) {
  using L = LinSmem<BN, F32S>;
  constexpr uint32_t kCols = 2 * BN;  // two f32 accumulators (a power of two >= 128)
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);  // 1024-byte aligned tiles
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* empty = full + L::kStages;
  uint64_t* acc_full = empty + L::kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (warp == 1) {
    tmem_alloc(tslot, kCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kLinEpiWarps);  // one arrival per epilogue warp
    }
    mbar_init_fence();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tslot;
  const int nkb = args.nkb_lo + args.nkb_hi;
  // A dependent kernel may be scheduled now; it waits for this grid's results
  // before reading them (griddepcontrol.wait above), and its CTAs only take an
  // SM once one of these has left it.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  bool timed_out = false;

  if (warp == 0) {
    if (lane == 0) {
      // TMA producer: a continuous K-block stream over this CTA's tiles. A may
      // be the previous kernel's output: with programmatic dependent launch
      // this kernel can start while that one finishes, so wait for it here
      // (a no-op without such a dependency).
      asm volatile("griddepcontrol.wait;" ::: "memory");
      int g = 0;
      for (int t = blockIdx.x; t < args.tiles && !timed_out; t += gridDim.x) {
        const int m0 = (t / args.tiles_n) * kLinBM, n0 = (t % args.tiles_n) * BN;
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int s = g % L::kStages;
          if (g >= L::kStages &&
              !mbar_wait_bounded(&empty[s], ((g / L::kStages) - 1) & 1, kLinWaitLimit)) {
            timed_out = true;
            break;
          }
          uint8_t* sa = smem + s * L::kStage;
          uint8_t* sb = sa + L::kA;
          mbar_arrive_expect_tx(&full[s], L::kStage);
          if (kb < args.nkb_lo) {
            tma_load_2d(sa, &map_a_lo, &full[s], kb * kLinBK, m0);
            tma_load_2d(sb, &map_w, &full[s], kb * kLinBK, n0);
          } else {
            const int kh = kb - args.nkb_lo;
            tma_load_2d(sa, &map_a_hi, &full[s], kh * kLinBK, m0);
            tma_load_2d(sb, &map_w, &full[s], args.k_lo + kh * kLinBK, n0);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // MMA issuer.
      constexpr uint32_t idesc = idesc_bf16_f32(kLinBM, BN);
      int g = 0, j = 0;
      for (int t = blockIdx.x; t < args.tiles && !timed_out; t += gridDim.x, ++j) {
        const int b = j & 1;
        if (j >= 2 && !mbar_wait_bounded(&acc_empty[b], ((j >> 1) - 1) & 1, kLinWaitLimit)) {
          timed_out = true;
          break;
        }
        tc_fence_after_sync();
        const uint32_t acc = tmem + static_cast<uint32_t>(b * BN);
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int s = g % L::kStages;
          if (!mbar_wait_bounded(&full[s], (g / L::kStages) & 1, kLinWaitLimit)) {
            timed_out = true;
            break;
          }
          tc_fence_after_sync();
          const uint32_t sa = smem_u32(smem + s * L::kStage);
          const uint32_t sb = sa + L::kA;
#pragma unroll
          for (int kk = 0; kk < kLinBK / 16; ++kk)
            tc_mma_bf16(acc, sdesc_k_sw128(sa + kk * 32), sdesc_k_sw128(sb + kk * 32), idesc,
                        (kb | kk) != 0 ? 1u : 0u);
          tc_commit(&empty[s]);  // the stage is free once these MMAs have read it
        }
        tc_commit(&acc_full[b]);  // the accumulator is final once all of them are done
      }
    }
  } else {
    // Epilogue warps 2..9: warp w reads TMEM lane quarter w % 4 (rows 32*(w%4) ..
    // +31 of a tile) and column half (w - 2) / 4 of the accumulator, 32 columns
    // per tcgen05.ld; its slice of the bias is staged in shared memory per tile.
    // A 32 x 32 result block goes out either through the warp's staging tiles
    // and one TMA store per output (lane r writes row r; 16-byte chunk q of a row
    // sits at chunk q ^ (r & 7) of a 128-byte f32 row and q ^ ((r >> 1) & 3) of a
    // 64-byte bf16 row, the layouts the maps' 128- and 64-byte swizzles read, so
    // the 32 lanes' 16-byte writes spread over all banks), or with direct stores.
    constexpr int kColsPerWarp = BN / 2;
    const int ew = warp - 2;
    const int quarter = warp & 3;
    const int c_begin = (ew >> 2) * kColsPerWarp;
    float* bias_s = reinterpret_cast<float*>(smem + L::kBias) + ew * kColsPerWarp;
    uint8_t* st32 = smem + L::kStaging + ew * (L::kStage32 + L::kStage16);
    uint8_t* st16 = st32 + L::kStage32;
    const bool f32_vec = args.y_f32 != nullptr && (args.ldy_f32 % 4) == 0 &&
                         (reinterpret_cast<uintptr_t>(args.y_f32) % 16) == 0;
    const bool bf_vec = args.y_bf16 != nullptr && (args.ldy_bf16 % 8) == 0 &&
                        (reinterpret_cast<uintptr_t>(args.y_bf16) % 16) == 0;
    const bool tma_out = args.tma_f32 || args.tma_bf16;
    int j = 0;
    for (int t = blockIdx.x; t < args.tiles; t += gridDim.x, ++j) {
      const int b = j & 1;
      const int m0 = (t / args.tiles_n) * kLinBM, n0 = (t % args.tiles_n) * BN;
      for (int c = lane; c < kColsPerWarp; c += 32) {
        const int n = n0 + c_begin + c;
        bias_s[c] = (args.bias != nullptr && n < args.N) ? __ldg(args.bias + n) : 0.f;
      }
      __syncwarp();
      const bool ok =
          __all_sync(0xffffffffu, mbar_wait_bounded(&acc_full[b], (j >> 1) & 1, kLinWaitLimit));
      if (!ok) {
        timed_out = true;
        break;
      }
      tc_fence_after_sync();
      const int row0 = m0 + quarter * 32;
      const uint32_t trow =
          tmem + static_cast<uint32_t>(b * BN) + (static_cast<uint32_t>(quarter * 32) << 16);
#pragma unroll 1
      for (int c0 = c_begin; c0 < c_begin + kColsPerWarp && n0 + c0 < args.N; c0 += 32) {
        float v[32];
        tmem_ld_32x32b_x32(trow + c0, v);
        const float4* bq = reinterpret_cast<const float4*>(bias_s + (c0 - c_begin));
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 bb = bq[q];
          v[4 * q] = activate<ACT>(__fadd_rn(v[4 * q], bb.x));
          v[4 * q + 1] = activate<ACT>(__fadd_rn(v[4 * q + 1], bb.y));
          v[4 * q + 2] = activate<ACT>(__fadd_rn(v[4 * q + 2], bb.z));
          v[4 * q + 3] = activate<ACT>(__fadd_rn(v[4 * q + 3], bb.w));
        }
        if (tma_out) {
          if (lane == 0) bulk_wait_read_all();  // the previous block has left the staging
          __syncwarp();
          if (F32S && args.tma_f32) {
            uint4* rowp = reinterpret_cast<uint4*>(st32 + lane * 128);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              rowp[q ^ (lane & 7)] =
                  make_uint4(__float_as_uint(v[4 * q]), __float_as_uint(v[4 * q + 1]),
                             __float_as_uint(v[4 * q + 2]), __float_as_uint(v[4 * q + 3]));
          }
          if (args.tma_bf16) {
            uint4* rowp = reinterpret_cast<uint4*>(st16 + lane * 64);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              rowp[q ^ ((lane >> 1) & 3)] = make_uint4(
                  pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                  pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (F32S && args.tma_f32) tma_store_2d(&map_y32, st32, n0 + c0, row0);
            if (args.tma_bf16) tma_store_2d(&map_y16, st16, n0 + c0, row0);
            bulk_commit();
          }
        }
        if (!args.tma_f32 || !args.tma_bf16) {
          LinearArgs direct = args;  // the outputs not written through TMA
          if (args.tma_f32) direct.y_f32 = nullptr;
          if (args.tma_bf16) direct.y_bf16 = nullptr;
          store_chunk32(direct, row0 + lane, n0 + c0, v, f32_vec, bf_vec);
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);  // this warp has drained its share
    }
    if (lane == 0) bulk_wait_all();  // every TMA store of this warp has completed
  }
  if (timed_out && args.status != nullptr) atomicOr(args.status, DLRM_FLAG_TIMEOUT);
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, kCols);
}

__global__ void f32_to_bf16_kernel(const float* __restrict__ x, int64_t ldx, int64_t rows,
                                   int64_t cols, uint16_t* __restrict__ y, int64_t ldy) {
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const float* xr = x + r * ldx;
    uint16_t* yr = y + r * ldy;
    for (int64_t c = threadIdx.x; c < cols; c += blockDim.x)
      yr[c] = __bfloat16_as_ushort(__float2bfloat16_rn(__ldg(xr + c)));
  }
}

// 2-D bf16 tensor map {cols, rows} with row pitch ld elements, box {64, box_rows},
// 128-byte swizzle; elements past the tensor read as zero.
cudaError_t encode_bf16_operand(CUtensorMap* map, const void* base, int64_t cols, int64_t rows,
                                int64_t ld, int box_rows) {
  const EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kLinBK), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int BN, int ACT, bool F32S>
cudaError_t run_linear(const CUtensorMap& a_lo, const CUtensorMap& a_hi, const CUtensorMap& w,
                       const CUtensorMap& y32, const CUtensorMap& y16, LinearArgs args, int sms,
                       cudaStream_t stream) {
  auto* fn = &linear_bf16_kernel<BN, ACT, F32S>;
  constexpr int smem = LinSmem<BN, F32S>::kTotal;
  cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(fn),
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  args.tiles_n = (args.N + BN - 1) / BN;
  const int64_t tiles = static_cast<int64_t>((args.M + kLinBM - 1) / kLinBM) * args.tiles_n;
  if (tiles > INT32_MAX) return cudaErrorInvalidValue;
  args.tiles = static_cast<int>(tiles);
  // one CTA per SM: the shared-memory ring and the 2 x BN TMEM columns size it
  const int grid = static_cast<int>(std::min<int64_t>(tiles, sms));
  // programmatic dependent launch: the prologue (TMEM allocation, barriers)
  // overlaps the tail of the kernel before it on the stream
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kLinThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fn, a_lo, a_hi, w, y32, y16, args);
}

template <int BN, bool F32S>
cudaError_t run_linear_act(int act, const CUtensorMap& a_lo, const CUtensorMap& a_hi,
                           const CUtensorMap& w, const CUtensorMap& y32, const CUtensorMap& y16,
                           const LinearArgs& args, int sms, cudaStream_t stream) {
  switch (act) {
    case DLRM_ACT_RELU:
      return run_linear<BN, DLRM_ACT_RELU, F32S>(a_lo, a_hi, w, y32, y16, args, sms, stream);
    case DLRM_ACT_SIGMOID:
      return run_linear<BN, DLRM_ACT_SIGMOID, F32S>(a_lo, a_hi, w, y32, y16, args, sms, stream);
    default:
      return run_linear<BN, DLRM_ACT_NONE, F32S>(a_lo, a_hi, w, y32, y16, args, sms, stream);
  }
}

// The instance with f32 output staging (and, at 256 columns, a 3-stage ring)
// only when the f32 output goes out through TMA.
template <int BN>
cudaError_t run_linear_bn(int act, const CUtensorMap& a_lo, const CUtensorMap& a_hi,
                          const CUtensorMap& w, const CUtensorMap& y32, const CUtensorMap& y16,
                          const LinearArgs& args, int sms, cudaStream_t stream) {
  return args.tma_f32 ? run_linear_act<BN, true>(act, a_lo, a_hi, w, y32, y16, args, sms, stream)
                      : run_linear_act<BN, false>(act, a_lo, a_hi, w, y32, y16, args, sms, stream);
}

// 2-D output map {N, M} with row pitch ld elements, box {32, 32}, written from a
// staging tile in the given swizzle layout.
cudaError_t encode_output(CUtensorMap* map, void* base, CUtensorMapDataType dt, int esz, int64_t N,
                          int64_t M, int64_t ld, CUtensorMapSwizzle swz) {
  const EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * esz};
  const cuuint32_t box[2] = {32, 32};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, dt, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         swz, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

int sm_count_current() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n;
}

// Tile width: the widest of 256, 128 whose tile count still covers every SM,
// else 64 (more, smaller tiles for small layers).
int choose_bn(int64_t M, int64_t N, int sms) {
#ifdef DLRM_LIN_FORCE_BN
  if (N > 64) return DLRM_LIN_FORCE_BN;
#endif
  const int64_t mt = (M + kLinBM - 1) / kLinBM;
  if (N <= 64) return 64;
  if (mt * ((N + 255) / 256) >= sms) return 256;
  if (mt * ((N + 127) / 128) >= sms) return 128;
  return 64;
}

bool is_aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace
}  // namespace dlrm

extern "C" {

DLRM_API int dlrm_linear_bf16(const uint16_t* a_lo, int64_t lda_lo, int64_t k_lo,
                              const uint16_t* a_hi, int64_t lda_hi, int64_t k_hi,
                              const uint16_t* w, int64_t ldw, const float* bias, int64_t M,
                              int64_t N, int act, float* y_f32, int64_t ldy_f32,
                              uint16_t* y_bf16, int64_t ldy_bf16, int32_t* status_dev,
                              dlrm_stream_t stream) {
  using namespace dlrm;
  if (a_lo == nullptr || w == nullptr) return DLRM_ERR_NULL;
  if (y_f32 == nullptr && y_bf16 == nullptr) return DLRM_ERR_NULL;
  if (k_hi > 0 && a_hi == nullptr) return DLRM_ERR_NULL;
  if (act < DLRM_ACT_NONE || act > DLRM_ACT_SIGMOID) return DLRM_ERR_ARG;
  if (M < 1 || N < 1 || k_lo < 1 || k_hi < 0) return DLRM_ERR_SHAPE;
  const int64_t K = k_lo + k_hi;
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return DLRM_ERR_SHAPE;
  if (lda_lo < k_lo || (k_hi > 0 && lda_hi < k_hi) || ldw < K) return DLRM_ERR_SHAPE;
  if ((y_f32 != nullptr && ldy_f32 < N) || (y_bf16 != nullptr && ldy_bf16 < N))
    return DLRM_ERR_SHAPE;
  if ((N + 63) / 64 > 65535) return DLRM_ERR_SHAPE;  // grid.y
  if (lda_lo % 8 != 0 || (k_hi > 0 && lda_hi % 8 != 0) || ldw % 8 != 0) return DLRM_ERR_ALIGN;
  if (k_hi > 0 && k_lo % 8 != 0) return DLRM_ERR_ALIGN;
  if (!is_aligned(a_lo, 16) || (k_hi > 0 && !is_aligned(a_hi, 16)) || !is_aligned(w, 16))
    return DLRM_ERR_ALIGN;
  if ((bias != nullptr && !is_aligned(bias, 4)) || (y_f32 != nullptr && !is_aligned(y_f32, 4)) ||
      (y_bf16 != nullptr && !is_aligned(y_bf16, 2)) ||
      (status_dev != nullptr && !is_aligned(status_dev, 4)))
    return DLRM_ERR_ALIGN;

  const int sms = sm_count_current();
  const int bn = choose_bn(M, N, sms);
  CUtensorMap ma_lo, ma_hi, mw;
  cudaError_t e = encode_bf16_operand(&ma_lo, a_lo, k_lo, M, lda_lo, kLinBM);
  if (e == cudaSuccess && k_hi > 0) e = encode_bf16_operand(&ma_hi, a_hi, k_hi, M, lda_hi, kLinBM);
  if (e == cudaSuccess) e = encode_bf16_operand(&mw, w, K, N, ldw, bn);
  if (e != cudaSuccess) return cuda_fail(e);
  if (k_hi == 0) ma_hi = ma_lo;  // never read

  LinearArgs args;
  args.bias = bias;
  args.y_f32 = y_f32;
  args.y_bf16 = y_bf16;
  args.ldy_f32 = ldy_f32;
  args.ldy_bf16 = ldy_bf16;
  args.M = static_cast<int>(M);
  args.N = static_cast<int>(N);
  args.k_lo = static_cast<int>(k_lo);
  args.nkb_lo = static_cast<int>((k_lo + kLinBK - 1) / kLinBK);
  args.nkb_hi = static_cast<int>((k_hi + kLinBK - 1) / kLinBK);
  args.status = status_dev;
  // Outputs whose rows are whole 16-byte units at 16-byte aligned addresses go
  // out through TMA stores; the others are written directly.
  CUtensorMap my32, my16;
  args.tma_f32 = y_f32 != nullptr && ldy_f32 % 4 == 0 && is_aligned(y_f32, 16);
  args.tma_bf16 = y_bf16 != nullptr && ldy_bf16 % 8 == 0 && is_aligned(y_bf16, 16);
  if (args.tma_f32)
    e = encode_output(&my32, y_f32, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, N, M, ldy_f32,
                      CU_TENSOR_MAP_SWIZZLE_128B);
  if (e == cudaSuccess && args.tma_bf16)
    e = encode_output(&my16, y_bf16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, M, ldy_bf16,
                      CU_TENSOR_MAP_SWIZZLE_64B);
  if (e != cudaSuccess) return cuda_fail(e);
  if (!args.tma_f32) my32 = mw;  // never read
  if (!args.tma_bf16) my16 = mw;  // never read
  auto* s = reinterpret_cast<cudaStream_t>(stream);
  switch (bn) {
    case 256: e = run_linear_bn<256>(act, ma_lo, ma_hi, mw, my32, my16, args, sms, s); break;
    case 128: e = run_linear_bn<128>(act, ma_lo, ma_hi, mw, my32, my16, args, sms, s); break;
    default: e = run_linear_bn<64>(act, ma_lo, ma_hi, mw, my32, my16, args, sms, s); break;
  }
  if (e != cudaSuccess) return cuda_fail(e);
  note_launch();
  return DLRM_OK;
}

DLRM_API int dlrm_f32_to_bf16(const float* x, int64_t ldx, int64_t rows, int64_t cols,
                              uint16_t* y, int64_t ldy, dlrm_stream_t stream) {
  using namespace dlrm;
  if (x == nullptr || y == nullptr) return DLRM_ERR_NULL;
  if (rows < 1 || cols < 1 || ldx < cols || ldy < cols) return DLRM_ERR_SHAPE;
  if (!is_aligned(x, 4) || !is_aligned(y, 2)) return DLRM_ERR_ALIGN;
  const int64_t blocks = std::min<int64_t>(rows, 148 * 32);
  const int threads = cols >= 256 ? 256 : static_cast<int>(((cols + 31) / 32) * 32);
  f32_to_bf16_kernel<<<static_cast<unsigned>(blocks), threads, 0,
                       reinterpret_cast<cudaStream_t>(stream)>>>(x, ldx, rows, cols, y, ldy);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  note_launch();
  return DLRM_OK;
}

}  // extern "C"
