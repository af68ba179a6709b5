// Persistent, pipelined register-load gather path (sm_100a), selectable with
// DLRM_PATH_PIPE for tables whose rows are whole 16-byte chunks.
//
// The plain gather pays, for every bag, three dependent trips to memory: the
// bag's bounds (offsets), then its row ids, then its rows. Here a lane group
// ("unit") of G lanes walks a long sequence of bags and keeps that chain out
// of the critical path: while it sums bag i it has already requested the row
// ids of bag i+1 and the bounds of bag i+2, so each bag exposes one memory
// latency (its rows), and U rows per lane (128-bit loads) are in flight at
// once. Rows past the first U of a bag are fetched in batches whose ids are
// requested one batch ahead. Each column is still summed from 0.0f in bag
// order with one rounding per step, so results are bit-identical to the
// sequential definition (and to the other paths).
//
// Blocks are persistent. In the fused kernel kPipeGatherWarps warps of units
// pool the bags of tile t into one of two feature buffers while kPipeDotWarps
// warps compute the interaction of the previous tile (fused_dot_warps); named
// barriers hand the buffers over.
#pragma once

#include "launch.h"
#include "persist_common.cuh"

namespace dlrm {

#ifndef DLRM_PIPE_ROWS
#define DLRM_PIPE_ROWS 8  // rows in flight per lane (16-byte chunks, one chunk per lane)
#endif
#ifndef DLRM_PIPE_GATHER_WARPS
#define DLRM_PIPE_GATHER_WARPS 12
#endif
#ifndef DLRM_PIPE_ONLY_THREADS
#define DLRM_PIPE_ONLY_THREADS 256
#endif
#ifndef DLRM_PIPE_ONLY_MIN_BLOCKS
#define DLRM_PIPE_ONLY_MIN_BLOCKS 2
#endif

constexpr int kPipeGatherWarps = DLRM_PIPE_GATHER_WARPS;
constexpr int kPipeDotWarps = 4;
constexpr int kPipeGatherOnlyThreads = DLRM_PIPE_ONLY_THREADS;

template <class LD, int G, int CPL, int POOL, bool FUSED>
struct PipeUnit {
  static constexpr int VEC = LD::VEC;
  // rows in flight per lane
  static constexpr int U = CPL == 1 ? DLRM_PIPE_ROWS : DLRM_PIPE_ROWS / 2;
  static constexpr int IPL = (U + G - 1) / G;  // row ids held per lane per batch
  using Raw = typename LD::Raw;
  using Elem = typename LD::Elem;

  int q, gbase;
  BagOrder<FUSED> order;
  BagPos cur, nxt;  // the bag being pooled and the next one (bounds ready)
  int nn_s, nn_e;   // raw offsets of the bag after that (in flight)
  int cid[IPL], nid[IPL];
  float cw[IPL], nw[IPL];
  bool oob, bad;

  __device__ __forceinline__ void load_ids(const BagParams& bp, const BagPos& p, int r0,
                                           int (&id)[IPL], float (&w)[IPL]) const {
#pragma unroll
    for (int j = 0; j < IPL; ++j) {
      const int slot = q + G * j;
      const int r = r0 + slot;
      const bool in = p.valid && slot < U && r < p.n;
      const int64_t at = static_cast<int64_t>(p.k) * bp.T + p.start + r;
      id[j] = in ? __ldg(bp.indices + at) : 0;
      if (POOL == kPoolWeighted) w[j] = in ? __ldg(bp.psw + at) : 0.f;
    }
  }

  __device__ __forceinline__ void start(const BagParams& bp) {
    order.first(cur);
    order.locate(cur, bp);
    load_ids(bp, cur, 0, cid, cw);
    order.next(cur, nxt);
    order.locate(nxt, bp);
    nn_s = nn_e = 0;
    oob = false;
    bad = cur.valid && cur.bad;
  }

  // Request the ids of the next bag and the offsets of the one after it.
  __device__ __forceinline__ void prefetch(const BagParams& bp) {
    load_ids(bp, nxt, 0, nid, nw);
    BagPos p;
    order.next(nxt, p);
    order.place(p);
    order.load_offsets(p, bp, nn_s, nn_e);
  }

  // Pool bag `cur` if it belongs to tile `lt` (fused) or exists (gather) and
  // hand the result to store(bag, chunk m, values). Every lane of the warp
  // calls this together: the loop runs to the warp's largest bag, so control
  // flow and shuffles stay warp-uniform. Returns false once no unit of the
  // warp has such a bag.
  template <class Store>
  __device__ __forceinline__ bool step(int lt, const TableParams& tp, const BagParams& bp, int D,
                                       Store&& store) {
    const bool active = cur.valid && (!FUSED || cur.lt == lt);
    if (!__any_sync(kFullMask, active)) return false;
    const int n = active ? cur.n : 0;
    const int nmax = __reduce_max_sync(kFullMask, n);
    const Elem* W = static_cast<const Elem*>(tp.w[cur.k]);
    const int rows_k = bp.check ? tp.rows[cur.k] : 0;
    bool colok[CPL];
#pragma unroll
    for (int m = 0; m < CPL; ++m) colok[m] = (q + G * m) * VEC < D;
    float acc[CPL][VEC];
#pragma unroll
    for (int m = 0; m < CPL; ++m)
#pragma unroll
      for (int e = 0; e < VEC; ++e) acc[m][e] = 0.f;
    int used = 0;
    int id[IPL];
    float w[IPL];
#pragma unroll
    for (int j = 0; j < IPL; ++j) {
      id[j] = cid[j];
      w[j] = cw[j];
    }
    bool prefetched = false;
    for (int c = 0; c < nmax; c += U) {
      Raw v[U][CPL];
      uint32_t use = 0;  // bit u: row c+u is summed
      float wt[POOL == kPoolWeighted ? U : 1];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int r = __shfl_sync(kFullMask, id[u / G], gbase + (u % G));
        if constexpr (POOL == kPoolWeighted)
          wt[u] = __shfl_sync(kFullMask, w[u / G], gbase + (u % G));
        bool ok = (c + u) < n;
        if (bp.check) {
          const bool in_range = static_cast<unsigned>(r) < static_cast<unsigned>(rows_k);
          oob |= ok && !in_range;
          ok = ok && in_range;
        }
        use |= ok ? (1u << u) : 0u;
        const Elem* row = W + static_cast<int64_t>(r) * D + q * VEC;
#pragma unroll
        for (int m = 0; m < CPL; ++m)
          if (ok && colok[m]) v[u][m] = LD::load(row + G * m * VEC);
      }
      if (active && !prefetched) {
        prefetch(bp);
        prefetched = true;
      }
      if (c + U < n) load_ids(bp, cur, c + U, id, w);  // next batch, one batch ahead
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (use & (1u << u)) {
#pragma unroll
          for (int m = 0; m < CPL; ++m)
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
              const float x = LD::get(v[u][m], e);
              if constexpr (POOL == kPoolSum) {
                acc[m][e] = __fadd_rn(acc[m][e], x);
              } else if constexpr (POOL == kPoolWeighted) {
                acc[m][e] = __fmaf_rn(wt[u], x, acc[m][e]);
              } else {
                acc[m][e] = (used == 0) ? x : ((x > acc[m][e]) ? x : acc[m][e]);
              }
            }
          ++used;
        }
      }
    }
    if (!active) return true;
    if (!prefetched) prefetch(bp);
    if (bp.mean && used > 0) {
      const float cnt = static_cast<float>(used);
#pragma unroll
      for (int m = 0; m < CPL; ++m)
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[m][e] = __fdiv_rn(acc[m][e], cnt);
    }
#pragma unroll
    for (int m = 0; m < CPL; ++m)
      if (colok[m]) store(cur, m, acc[m]);
    // rotate: the next bag's ids and the offsets after it are already in flight
    cur = nxt;
#pragma unroll
    for (int j = 0; j < IPL; ++j) {
      cid[j] = nid[j];
      cw[j] = nw[j];
    }
    order.next(cur, nxt);
    order.place(nxt);
    BagOrder<FUSED>::set_bounds(nxt, nn_s, nn_e, bp.T);
    bad |= cur.valid && cur.bad;
    return true;
  }
};

template <class LD, int G, int CPL, int POOL, bool FUSED>
__device__ __forceinline__ void init_pipe_unit(PipeUnit<LD, G, CPL, POOL, FUSED>& U, int units,
                                               int B, int F, int S, int my_tiles) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = warp * (32 / G) + lane / G;
  U.q = lane % G;
  U.gbase = lane - U.q;
  U.order = BagOrder<FUSED>{B, F, S, units, u, my_tiles};
}

__device__ __forceinline__ void pipe_report(const BagParams& bp, bool oob, bool bad) {
  if (bp.status != nullptr) {
    const int flags = (oob ? DLRM_FLAG_INDEX_OOB : 0) | (bad ? DLRM_FLAG_OFFSETS : 0);
    if (flags) atomicOr(bp.status, flags);
  }
}

template <int VEC>
__device__ __forceinline__ void store_chunk(float* p, const float (&a)[VEC]) {
  if constexpr (VEC == 1) {
    *p = a[0];
  } else {
    store_vec_f32<VEC>(p, a);
  }
}

// --------------------------------------------------------------------------
// Gather only: persistent blocks of units writing pooled rows to `out`.
template <class LD, int G, int CPL, int POOL>
__global__ void __launch_bounds__(kPipeGatherOnlyThreads, DLRM_PIPE_ONLY_MIN_BLOCKS)
    pipe_embbag_kernel(const __grid_constant__ TableParams tp, const BagParams bp, int B, int F,
                       int D, float* __restrict__ out) {
  constexpr int VEC = LD::VEC;
  constexpr int units = kPipeGatherOnlyThreads / G;
  PipeUnit<LD, G, CPL, POOL, false> U;
  init_pipe_unit(U, units, B, F, 1, 0);
  U.start(bp);
  auto store = [&](const BagPos& bg, int m, const float (&a)[VEC]) {
    store_chunk<VEC>(out + (static_cast<int64_t>(bg.b) * F + bg.k) * D + (U.q + G * m) * VEC, a);
  };
  while (U.step(0, tp, bp, D, store)) {
  }
  if (U.q == 0) pipe_report(bp, U.oob, U.bad);
}

// --------------------------------------------------------------------------
// Fused: gather warps pool tile lt into feature buffer lt&1 while dot warps
// finish tile lt-1; each tile holds S consecutive samples.
template <class LD, int G, int CPL, int POOL>
__global__ void __launch_bounds__((kPipeGatherWarps + kPipeDotWarps) * 32, 1)
    pipe_fused_kernel(const __grid_constant__ TableParams tp, const BagParams bp,
                      const float* __restrict__ dense, int B, int F, int D, int S, int lq,
                      float* __restrict__ pooled_out, float* __restrict__ inter_out,
                      int concat_dense) {
  extern __shared__ __align__(16) float feat[];
  constexpr int NT = (kPipeGatherWarps + kPipeDotWarps) * 32;
  constexpr int VEC = LD::VEC;
  const FeatLayout Lf = FeatLayout::make(F, D);
  const int64_t sample_floats = Lf.floats_per_sample();
  const int my_tiles = block_tiles(B, S);
  const int warp = threadIdx.x >> 5;

  if (warp < kPipeGatherWarps) {
    constexpr int units = kPipeGatherWarps * 32 / G;
    PipeUnit<LD, G, CPL, POOL, true> U;
    init_pipe_unit(U, units, B, F, S, my_tiles);
    U.start(bp);
    for (int lt = 0; lt < my_tiles; ++lt) {
      const int p = lt & 1;
      if (lt >= 2) named_bar_sync(kBarFree0 + p, NT);
      float* fb = feat + p * S * sample_floats;
      const int64_t b0 =
          (static_cast<int64_t>(blockIdx.x) + static_cast<int64_t>(lt) * gridDim.x) * S;
      auto store = [&](const BagPos& bg, int m, const float (&a)[VEC]) {
        const int s = static_cast<int>(bg.b - b0);
        const int col = (U.q + G * m) * VEC;
        store_chunk<VEC>(fb + s * sample_floats + (1 + bg.k) * Lf.Dp + col, a);
        if (pooled_out)
          store_chunk<VEC>(pooled_out + (static_cast<int64_t>(bg.b) * F + bg.k) * D + col, a);
      };
      while (U.step(lt, tp, bp, D, store)) {
      }
      __syncwarp();
      named_bar_arrive(kBarReady0 + p, NT);
    }
    if (U.q == 0) pipe_report(bp, U.oob, U.bad);
  } else {
    fused_dot_warps<kPipeGatherWarps, kPipeDotWarps>(feat, Lf, dense, B, D, S, lq, my_tiles,
                                                     inter_out, concat_dense);
  }
}

// --------------------------------------------------------------------------
// Host-side dispatch.

template <class LD, int G, int CPL, int POOL>
cudaError_t run_pipe_gather(const PipeLaunch& a) {
  auto* fn = &pipe_embbag_kernel<LD, G, CPL, POOL>;
  int per_sm = 0;
  cudaError_t e =
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kPipeGatherOnlyThreads, 0);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int units = kPipeGatherOnlyThreads / G;
  const int64_t work = (static_cast<int64_t>(a.B) * a.F + units - 1) / units;
  const int64_t grid = std::min<int64_t>(static_cast<int64_t>(per_sm) * a.sms, work);
  fn<<<static_cast<unsigned>(grid), kPipeGatherOnlyThreads, 0, a.stream>>>(*a.tp, a.bp, a.B, a.F,
                                                                           a.D, a.out);
  return cudaGetLastError();
}

template <class LD, int G, int CPL, int POOL>
cudaError_t run_pipe_fused(const PipeLaunch& a) {
  auto* fn = &pipe_fused_kernel<LD, G, CPL, POOL>;
  constexpr int NT = (kPipeGatherWarps + kPipeDotWarps) * 32;
  if (a.smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(fn),
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(a.smem));
    if (e != cudaSuccess) return e;
  }
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, NT, a.smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int64_t ntiles = (static_cast<int64_t>(a.B) + a.S - 1) / a.S;
  const int64_t grid = std::min<int64_t>(static_cast<int64_t>(per_sm) * a.sms, ntiles);
  fn<<<static_cast<unsigned>(grid), NT, a.smem, a.stream>>>(*a.tp, a.bp, a.dense, a.B, a.F, a.D,
                                                             a.S, a.lq, a.pooled_out,
                                                             a.inter_out, a.concat_dense);
  return cudaGetLastError();
}

#define DLRM_PIPE_POOLS(RUN, LD_, G_, C_, a)                                      \
  do {                                                                          \
    if ((a).pool == kPoolSum) return RUN<LD_, G_, C_, kPoolSum>(a);             \
    if ((a).pool == kPoolWeighted) return RUN<LD_, G_, C_, kPoolWeighted>(a);   \
    return RUN<LD_, G_, C_, kPoolMax>(a);                                       \
  } while (0)

#define DLRM_PIPE_DISPATCH(RUN, LD_, a)                                          \
  do {                                                                          \
    if ((a).cpl == 2) DLRM_PIPE_POOLS(RUN, LD_, 32, 2, a);                      \
    switch ((a).G) {                                                            \
      case 4: DLRM_PIPE_POOLS(RUN, LD_, 4, 1, a);                               \
      case 8: DLRM_PIPE_POOLS(RUN, LD_, 8, 1, a);                               \
      case 16: DLRM_PIPE_POOLS(RUN, LD_, 16, 1, a);                             \
      default: DLRM_PIPE_POOLS(RUN, LD_, 32, 1, a);                             \
    }                                                                           \
  } while (0)

}  // namespace dlrm
