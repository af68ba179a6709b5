// Gather and fused kernel templates of the DLRMv1 sparse/interaction stage
// (sm_100a). Each inst_*.cu file instantiates them for one row loader.
#pragma once

#include "interact_common.cuh"
#include "launch.h"

namespace dlrm {

// Rows each lane fetches before consuming any (per column chunk), and the
// blocks per SM the register allocation must allow.
#ifndef DLRM_ROWS_IN_FLIGHT
#define DLRM_ROWS_IN_FLIGHT 8
#endif
#ifndef DLRM_GATHER_MIN_BLOCKS
#define DLRM_GATHER_MIN_BLOCKS 8
#endif
constexpr int kRowsInFlight = DLRM_ROWS_IN_FLIGHT;
constexpr int kGatherMinBlocks = DLRM_GATHER_MIN_BLOCKS;
constexpr int kFusedMinBlocks = DLRM_FUSED_MIN_BLOCKS;

// --------------------------------------------------------------------------
// Gather: one lane group of G lanes per bag (b, k); bag id u = b*F + k, so
// consecutive groups write consecutive pooled vectors
// (embedding_bag.rs, multi-table section of the pages: one launch, all tables).
template <class LD, int G, int CPL, int POOL>
__global__ void __launch_bounds__(kBlockThreads, kGatherMinBlocks)
    embbag_kernel(const __grid_constant__ TableParams tp, const BagParams bp, int B, int F, int D,
                  int ncolwin, float* __restrict__ out) {
  constexpr int VEC = LD::VEC;
  constexpr int U = CPL == 1 ? kRowsInFlight : kRowsInFlight / 2;
  constexpr int kGroups = kBlockThreads / G;
  using Elem = typename LD::Elem;
  const int lane = threadIdx.x & 31;
  const int q = lane % G;
  const int gbase = lane - q;
  const int64_t bag = static_cast<int64_t>(blockIdx.x) * kGroups + threadIdx.x / G;
  const bool active = bag < static_cast<int64_t>(B) * F;
  if (__all_sync(kFullMask, !active)) return;

  const int b = active ? static_cast<int>(bag / F) : 0;
  const int k = active ? static_cast<int>(bag - static_cast<int64_t>(b) * F) : 0;
  int start = 0, n = 0;
  bool bad = false;
  if (active) bag_bounds(bp, B, k, b, start, n, bad);
  const int nmax = __reduce_max_sync(kFullMask, n);
  const Elem* W = static_cast<const Elem*>(tp.w[k]);
  const int32_t* idx_seg = bp.indices + static_cast<int64_t>(k) * bp.T;
  const float* w_seg = bp.psw ? bp.psw + static_cast<int64_t>(k) * bp.T : nullptr;
  const int rows_k = bp.check ? tp.rows[k] : 0;
  bool oob = false;
  float* orow = out + (static_cast<int64_t>(b) * F + k) * D;

  for (int w = 0; w < ncolwin; ++w) {
    const int col0 = w * (G * CPL * VEC);
    float acc[CPL][VEC];
    const int used = pool_bag<LD, G, CPL, U, POOL>(W, rows_k, bp.check, idx_seg, w_seg, start,
                                                   n, nmax, D, col0, q, gbase, acc, oob);
    if (bp.mean) finish_mean(acc, used);
    if (active) {
#pragma unroll
      for (int m = 0; m < CPL; ++m) {
        const int col = col0 + (q + G * m) * VEC;
        if (col < D) store_floats<VEC>(orow + col, acc[m]);
      }
    }
  }
  if (bp.status != nullptr) {
    const int flags = (oob ? DLRM_FLAG_INDEX_OOB : 0) | (bad ? DLRM_FLAG_OFFSETS : 0);
    if (flags) atomicOr(bp.status, flags);
  }
}

// How phase 1 of the fused kernel orders the bags: slot j of a round is bag j
// (fixed-stride bags), the bags are taken in sorted runs as described below
// (the general entry point, bags of any lengths), or bp.balance chooses.
enum FusedOrder { kOrderNone = 0, kOrderRuns = 1, kOrderByFlag = 2 };

// Phase 1 of the fused kernel: the block's bags (s, k) -> feature row k + 1
// (and pooled_out); every lane group runs the same number of rounds.
// Bags of different lengths: a warp runs to its longest bag and the block to
// its slowest warp. So the block's bags are taken in runs of 32; a warp
// reads the bounds of the run that holds its slots, sorts the run longest
// first (key: length, then bag number, so keys are unique and equal lengths
// order by bag number, higher first; a run whose bags all have one length is
// not sorted and keeps ascending bag order), and the rounds walk the sorted
// runs in alternating direction: the lane groups of a warp get bags of
// similar length, and a warp that drew long bags in one round draws short
// ones in the next. Every warp sorts the same runs the same way, so no block-wide
// barrier is needed; each warp keeps its sorted run in its own 96 ints of
// shared memory after the features (rank r: bag, start, length).
template <class LD, int G, int CPL, int POOL, int ORDER>
__device__ __forceinline__ void fused_gather_rounds(const TableParams& tp, const BagParams& bp,
                                                    float* feat, const FeatLayout& Lf, int B,
                                                    int F, int D, int ncolwin, int S, int64_t b0,
                                                    int ntasks, int rounds,
                                                    float* __restrict__ pooled_out, bool& oob,
                                                    bool& bad_any) {
  constexpr int VEC = LD::VEC;
  constexpr int U = CPL == 1 ? kRowsInFlight : kRowsInFlight / 2;
  constexpr int kGroups = kBlockThreads / G;
  using Elem = typename LD::Elem;
  const int lane = threadIdx.x & 31;
  const int q = lane % G;
  const int gbase = lane - q;
  const int64_t sample_floats = Lf.floats_per_sample();
  const int group = static_cast<int>(threadIdx.x) / G;
  const bool ordered = ORDER == kOrderRuns || (ORDER == kOrderByFlag && bp.balance);
  for (int rd = 0; rd < rounds; ++rd) {
    const int slot = rd * kGroups + ((ordered && (rd & 1)) ? kGroups - 1 - group : group);
    const bool active = slot < ntasks;
    int task = slot, start = 0, n = 0;
    if (ordered) {
      // all slots of a warp in a round lie in one run of 32 (warp-uniform);
      // the run is (re)sorted when it differs from the previous round's
      const int g0 = static_cast<int>(threadIdx.x - lane) / G;
      const auto run_of = [&](int r) {
        return (r * kGroups + ((r & 1) ? kGroups - 1 - g0 : g0)) >> 5;
      };
      const int run = run_of(rd);
      const int prev = rd == 0 ? -1 : run_of(rd - 1);
      int* run_sorted = reinterpret_cast<int*>(feat + static_cast<int64_t>(S) * sample_floats) +
                        (threadIdx.x >> 5) * 96;
      if (run != prev) {
        const int t = (run << 5) + lane;
        int st = 0, len = 0;
        unsigned key = 0;  // below every real key: empty slots sort last
        if (t < ntasks) {
          const int s = t / F;
          bool bad;
          bag_bounds(bp, B, t - s * F, static_cast<int>(b0 + s), st, len, bad);
          bad_any |= bad;
          key = ((static_cast<unsigned>(min(len, kSortLenMax)) + 1u) << kSortTaskBits) |
                static_cast<unsigned>(t);
        }
        const int len0 = __shfl_sync(kFullMask, len, 0);
        if (!__all_sync(kFullMask, t >= ntasks || len == len0)) key = warp_sort_desc(key, lane);
        const int tr = static_cast<int>(key & ((1u << kSortTaskBits) - 1u));
        const int st_r = __shfl_sync(kFullMask, st, tr & 31);
        const int len_r = __shfl_sync(kFullMask, len, tr & 31);
        __syncwarp();  // the previous run's reads are done
        run_sorted[lane] = tr;
        run_sorted[32 + lane] = st_r;
        run_sorted[64 + lane] = len_r;
        __syncwarp();
      }
      if (active) {
        const int r = slot & 31;
        task = run_sorted[r];
        start = run_sorted[32 + r];
        n = run_sorted[64 + r];
      }
    } else if (active) {
      const int s = task / F;
      bool bad = false;
      bag_bounds(bp, B, task - s * F, static_cast<int>(b0 + s), start, n, bad);
      bad_any |= bad;
    }
    const int s = active ? task / F : 0;
    const int k = active ? task - s * F : 0;
    const int nmax = __reduce_max_sync(kFullMask, n);
    const Elem* W = static_cast<const Elem*>(tp.w[k]);
    const int32_t* idx_seg = bp.indices + static_cast<int64_t>(k) * bp.T;
    const float* w_seg = bp.psw ? bp.psw + static_cast<int64_t>(k) * bp.T : nullptr;
    const int rows_k = bp.check ? tp.rows[k] : 0;
    float* frow = feat + s * sample_floats + (1 + k) * Lf.Dp;
    float* prow = pooled_out ? pooled_out + ((b0 + s) * F + k) * static_cast<int64_t>(D)
                             : nullptr;
    for (int w = 0; w < ncolwin; ++w) {
      const int col0 = w * (G * CPL * VEC);
      float acc[CPL][VEC];
      const int used = pool_bag<LD, G, CPL, U, POOL>(W, rows_k, bp.check, idx_seg, w_seg, start,
                                                     n, nmax, D, col0, q, gbase, acc, oob);
      if (bp.mean) finish_mean(acc, used);
      if (active) {
#pragma unroll
        for (int m = 0; m < CPL; ++m) {
          const int col = col0 + (q + G * m) * VEC;
          if (col < D) {
            if constexpr (VEC == 1) {
              frow[col] = acc[m][0];
            } else {
              store_floats<VEC>(frow + col, acc[m]);
            }
            if (prow) store_floats<VEC>(prow + col, acc[m]);
          }
        }
      }
    }
  }
}

// --------------------------------------------------------------------------
// Fused: each block owns S consecutive samples. Phase 1 gathers their S*F
// bags straight into shared memory (and, if asked, to pooled_out) next to the
// dense rows; phase 2 computes the dots from shared memory. Only pooled_out
// and inter_out are written to global memory.
template <class LD, int G, int CPL, int POOL, int ORDER>
__global__ void __launch_bounds__(kBlockThreads, kFusedMinBlocks)
    fused_kernel(const __grid_constant__ TableParams tp, const BagParams bp,
                 const float* __restrict__ dense, int B, int F, int D, int ncolwin, int S, int lq,
                 float* __restrict__ pooled_out, float* __restrict__ inter_out, int concat_dense) {
  constexpr int kGroups = kBlockThreads / G;
  extern __shared__ __align__(16) float feat[];
  const FeatLayout Lf = FeatLayout::make(F, D);
  const int64_t b0 = static_cast<int64_t>(blockIdx.x) * S;
  const int S_here = (B - b0 < S) ? static_cast<int>(B - b0) : S;
  const int64_t sample_floats = Lf.floats_per_sample();

  // dense rows -> feature row 0 with asynchronous copies (16-byte ones when the
  // pointer allows), waited for before the dot phase: the copying warp starts
  // its bags at once instead of a memory round trip later
  const bool dense_vec = ((D & 3) == 0) && ((reinterpret_cast<uintptr_t>(dense) & 15) == 0);
  for (int s = 0; s < S_here; ++s) {
    const float* src = dense + (b0 + s) * D;
    float* dst = feat + s * sample_floats;
    if (dense_vec) {
      for (int c = threadIdx.x; c < (D >> 2); c += blockDim.x) cp_async16(dst + 4 * c, src + 4 * c);
    } else {
      for (int c = threadIdx.x; c < D; c += blockDim.x) cp_async4(dst + c, src + c);
    }
  }
  cp_async_commit();
  zero_feature_padding(feat, Lf, D, S_here, threadIdx.x, blockDim.x);

  // bags (s, k) -> feature row k + 1; every group runs the same number of rounds
  bool oob = false, bad_any = false;
  const int ntasks = S_here * F;
  const int rounds = (S * F + kGroups - 1) / kGroups;
  fused_gather_rounds<LD, G, CPL, POOL, ORDER>(tp, bp, feat, Lf, B, F, D, ncolwin, S, b0, ntasks,
                                                rounds, pooled_out, oob, bad_any);
  if (bp.status != nullptr) {
    const int flags = (oob ? DLRM_FLAG_INDEX_OOB : 0) | (bad_any ? DLRM_FLAG_OFFSETS : 0);
    if (flags) atomicOr(bp.status, flags);
  }
  cp_async_wait<0>();  // this thread's dense copies have landed
  __syncthreads();

  const int64_t P = static_cast<int64_t>(Lf.F1) * (Lf.F1 - 1) / 2;
  const int64_t row_stride = concat_dense ? D + P : P;
  if (concat_dense) {
    for (int s = 0; s < S_here; ++s) {
      const float* src = feat + s * sample_floats;
      float* dst = inter_out + (b0 + s) * row_stride;
      for (int d = threadIdx.x; d < D; d += blockDim.x) dst[d] = src[d];
    }
  }
  dots_from_smem(feat, Lf, S_here, lq, inter_out, b0, row_stride, concat_dense ? D : 0,
                 threadIdx.x, blockDim.x);
}

// --------------------------------------------------------------------------
// Host-side dispatch over (G, CPL, POOL) for one loader.

template <class LD, int G, int CPL, int POOL>
cudaError_t run_gather(const GatherLaunch& a) {
  const int groups = kBlockThreads / G;
  const int64_t grid = (static_cast<int64_t>(a.B) * a.F + groups - 1) / groups;
  if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
  embbag_kernel<LD, G, CPL, POOL><<<static_cast<unsigned>(grid), kBlockThreads, 0, a.stream>>>(
      *a.tp, a.bp, a.B, a.F, a.D, a.shape.ncolwin, a.out);
  return cudaGetLastError();
}

template <class LD, int G, int CPL, int POOL>
cudaError_t run_fused(const FusedLaunch& a) {
  // Bags in length-sorted runs (general entry point) or in order (fixed
  // stride). Measured on B200: f32 rows run faster with one instance per
  // order (c3 52.6 -> 51.7 us, c5 1.67 -> 1.61 ms), bf16 rows with the
  // choice made at run time in one instance (c3 47.1 -> 44.4 us, c5 1.34 ->
  // 1.30 ms; register allocation at the 64-register cap).
  void (*fn)(const TableParams, const BagParams, const float*, int, int, int, int, int, int,
             float*, float*, int);
  if constexpr (sizeof(typename LD::Elem) == 2) {
    fn = &fused_kernel<LD, G, CPL, POOL, kOrderByFlag>;
  } else {
    fn = a.g.bp.balance ? &fused_kernel<LD, G, CPL, POOL, kOrderRuns>
                        : &fused_kernel<LD, G, CPL, POOL, kOrderNone>;
  }
  if (a.smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(fn),
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(a.smem));
    if (e != cudaSuccess) return e;
  }
  const int64_t grid = (static_cast<int64_t>(a.g.B) + a.S - 1) / a.S;
  fn<<<static_cast<unsigned>(grid), kBlockThreads, a.smem, a.g.stream>>>(
      *a.g.tp, a.g.bp, a.dense, a.g.B, a.g.F, a.g.D, a.g.shape.ncolwin, a.S, a.lq, a.pooled_out,
      a.inter_out, a.concat_dense);
  return cudaGetLastError();
}

// Calls F<LD, G, CPL, POOL>(arg) for the runtime (G, CPL, POOL).
#define DLRM_DISPATCH_SHAPES(RUN, LD, arg, shape, pool)                                \
  do {                                                                                 \
    const int G_ = (shape).G, C_ = (shape).cpl, P_ = (pool);                           \
    if (C_ == 2) {                                                                     \
      if (P_ == kPoolSum) return RUN<LD, 32, 2, kPoolSum>(arg);                        \
      if (P_ == kPoolWeighted) return RUN<LD, 32, 2, kPoolWeighted>(arg);              \
      return RUN<LD, 32, 2, kPoolMax>(arg);                                            \
    }                                                                                  \
    switch (G_) {                                                                      \
      case 4:                                                                          \
        if (P_ == kPoolSum) return RUN<LD, 4, 1, kPoolSum>(arg);                       \
        if (P_ == kPoolWeighted) return RUN<LD, 4, 1, kPoolWeighted>(arg);             \
        return RUN<LD, 4, 1, kPoolMax>(arg);                                           \
      case 8:                                                                          \
        if (P_ == kPoolSum) return RUN<LD, 8, 1, kPoolSum>(arg);                       \
        if (P_ == kPoolWeighted) return RUN<LD, 8, 1, kPoolWeighted>(arg);             \
        return RUN<LD, 8, 1, kPoolMax>(arg);                                           \
      case 16:                                                                         \
        if (P_ == kPoolSum) return RUN<LD, 16, 1, kPoolSum>(arg);                      \
        if (P_ == kPoolWeighted) return RUN<LD, 16, 1, kPoolWeighted>(arg);            \
        return RUN<LD, 16, 1, kPoolMax>(arg);                                          \
      default:                                                                         \
        if (P_ == kPoolSum) return RUN<LD, 32, 1, kPoolSum>(arg);                      \
        if (P_ == kPoolWeighted) return RUN<LD, 32, 1, kPoolWeighted>(arg);            \
        return RUN<LD, 32, 1, kPoolMax>(arg);                                          \
    }                                                                                  \
  } while (0)

#define DLRM_INSTANTIATE_LOADER(LD, NAME)                                              \
  cudaError_t launch_gather_##NAME(const GatherLaunch& a) {                            \
    DLRM_DISPATCH_SHAPES(run_gather, LD, a, a.shape, a.pool);                          \
  }                                                                                    \
  cudaError_t launch_fused_##NAME(const FusedLaunch& a) {                              \
    DLRM_DISPATCH_SHAPES(run_fused, LD, a, a.g.shape, a.g.pool);                       \
  }

}  // namespace dlrm
