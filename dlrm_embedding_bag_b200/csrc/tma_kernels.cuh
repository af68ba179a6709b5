// TMA gather path of the DLRMv1 sparse/interaction stage (sm_100a).
//
// Rows are fetched with the tensor-map tile::gather4 load: one instruction
// brings four arbitrary rows of a table into shared memory and reports their
// bytes on an mbarrier. A lane group ("unit") of G lanes pools one bag at a
// time; lane q owns the 16-byte chunks q, q+G, ... (CPL of them) of a row.
// Each unit keeps its own ring of kTmaBufs segment buffers (kTmaSegRows rows
// each) in flight ahead of the segment it is summing, so the bytes in flight
// cost shared memory, not registers. Measured on B200, the gather4 stream
// reaches the HBM copy rate only with about 32 independently issuing units per
// SM, so units are narrow (G = 8 for rows up to 256 bytes) and a block holds
// 32 of them. Row ids (and per-sample weights) of the next segment are fetched
// one step ahead with ordinary loads and published in shared memory for the
// issuing lane and the summing lanes; bag bounds are fetched one bag ahead.
//
// Blocks are persistent. In the fused kernel, gather warps pool the bags of
// tile t into one of two feature buffers while dot warps compute the
// interaction of the previous tile from the other; named barriers hand the
// buffers over (READY: gather -> dot, FREE: dot -> gather).
//
// Every mbarrier wait is bounded (about 0.1 s); a wait that runs out raises
// DLRM_FLAG_TIMEOUT in the status word (when one is given), the unit stops
// waiting from then on, and the kernel carries on, so it always terminates.
#pragma once

#include "interact_common.cuh"
#include "launch.h"
#include "persist_common.cuh"
#include "tma_common.cuh"

namespace dlrm {

constexpr int kTmaQuadsPerSeg = 2;
constexpr int kTmaSegRows = 4 * kTmaQuadsPerSeg;
constexpr int kTmaBufs = 2;
constexpr int kTmaGatherWarps = 8;
constexpr int kTmaDotWarps = 4;
constexpr long long kTmaWaitLimit = 200000000LL;  // clock cycles, about 0.1 s

// What one issued segment holds; written by the unit before it issues.
struct SegMeta {
  int valid;  // 0 marks the end of the unit's sequence
  int lt;     // local tile index (fused kernel), else 0
  int b, k;   // sample and table of the bag
  int n;      // bag length
  int r0;     // first bag row held by this segment
  int nrows;  // rows held (0 for an empty bag)
  int pad;
};

// Shared-memory carve-up of one block.
struct TmaSmem {
  int units;        // units per block
  int box_bytes;    // bytes of one table row (the tensor map's box)
  int quad_stride;  // bytes between the 4-row quads of a buffer (multiple of 128)
  int buf_bytes;    // bytes of one segment buffer
  int64_t bars_off, meta_off, ids_off, wts_off, feat_off, total;
  __host__ __device__ static TmaSmem make(int G, int box_bytes, int64_t feat_bytes) {
    TmaSmem s;
    s.units = kTmaGatherWarps * (32 / G);
    s.box_bytes = box_bytes;
    s.quad_stride = ((4 * box_bytes + 127) / 128) * 128;
    s.buf_bytes = kTmaQuadsPerSeg * s.quad_stride;
    const int64_t nb = static_cast<int64_t>(s.units) * kTmaBufs;
    s.bars_off = nb * s.buf_bytes;
    s.meta_off = s.bars_off + nb * 8;
    s.ids_off = s.meta_off + nb * static_cast<int64_t>(sizeof(SegMeta));
    s.wts_off = s.ids_off + nb * kTmaSegRows * 4;
    s.feat_off = ((s.wts_off + nb * kTmaSegRows * 4 + 15) / 16) * 16;
    s.total = s.feat_off + feat_bytes;
    return s;
  }
};

template <int G, int CPL, int POOL, int ESZ, bool FUSED>
struct TmaUnit {
  static constexpr int VEC = 16 / ESZ;                   // table elements per 16-byte chunk
  static constexpr int IPL = (kTmaSegRows + G - 1) / G;  // row ids per lane

  unsigned char* ring;
  uint64_t* bars;
  SegMeta* meta;
  int32_t* ids;
  float* wts;
  int buf_bytes, quad_stride, box_bytes;
  unsigned mask;
  int q;
  BagOrder<FUSED> order;
  // issue side
  BagPos cur, ahead;  // the bag being issued, and the next one (bounds in flight)
  int r0;             // next row of `cur` to issue
  int pre_id[IPL];
  float pre_w[IPL];
  // consume side
  int c;
  uint32_t phase;
  float acc[CPL][VEC];
  int used;
  bool oob, bad, timeout;

  __device__ __forceinline__ bool chunk_ok(int m) const { return (q + G * m) * 16 < box_bytes; }

  __device__ __forceinline__ void prefetch_rows(const BagParams& bp) {
#pragma unroll
    for (int j = 0; j < IPL; ++j) {
      const int slot = q + G * j;
      const int r = r0 + slot;
      const bool in = cur.valid && slot < kTmaSegRows && r < cur.n;
      const int64_t at = static_cast<int64_t>(cur.k) * bp.T + cur.start + r;
      pre_id[j] = in ? __ldg(bp.indices + at) : 0;
      if (POOL == kPoolWeighted) pre_w[j] = in ? __ldg(bp.psw + at) : 0.f;
    }
  }

  __device__ __forceinline__ void start(const BagParams& bp) {
    order.first(cur);
    order.locate(cur, bp);
    order.next(cur, ahead);
    order.locate(ahead, bp);
    r0 = 0;
    bad = cur.valid && cur.bad;
    prefetch_rows(bp);
    c = 0;
    phase = 0;
    used = 0;
    oob = timeout = false;
  }

  __device__ __forceinline__ void advance(const BagParams& bp) {
    if (!cur.valid) return;
    if (r0 + kTmaSegRows < cur.n) {
      r0 += kTmaSegRows;
    } else {
      cur = ahead;  // its bounds were requested one bag ago
      order.next(cur, ahead);
      order.locate(ahead, bp);
      r0 = 0;
      bad |= cur.valid && cur.bad;
    }
    prefetch_rows(bp);
  }

  // Publish the pending segment into buffer `buf`, launch its loads, advance.
  __device__ __forceinline__ void issue(int buf, const TmaParams& tp, const BagParams& bp) {
    const int nrows = cur.valid ? min(kTmaSegRows, cur.n - r0) : 0;
    if (q == 0) {
      SegMeta v;
      v.valid = cur.valid;
      v.lt = cur.lt;
      v.b = cur.b;
      v.k = cur.k;
      v.n = cur.n;
      v.r0 = r0;
      v.nrows = nrows;
      v.pad = 0;
      meta[buf] = v;
    }
#pragma unroll
    for (int j = 0; j < IPL; ++j) {
      const int slot = q + G * j;
      if (slot < kTmaSegRows) {
        ids[buf * kTmaSegRows + slot] = pre_id[j];
        if (POOL == kPoolWeighted) wts[buf * kTmaSegRows + slot] = pre_w[j];
      }
    }
    __syncwarp(mask);
    if (q == 0 && nrows > 0) {
      const int nq = (nrows + 3) / 4;
      const int32_t* id = ids + buf * kTmaSegRows;
      uint64_t* bar = bars + buf;
      mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nq * 4 * box_bytes));
      for (int qd = 0; qd < nq; ++qd) {
        const int r = 4 * qd;
        const int y0 = id[r];
        const int y1 = (r + 1 < nrows) ? id[r + 1] : y0;
        const int y2 = (r + 2 < nrows) ? id[r + 2] : y0;
        const int y3 = (r + 3 < nrows) ? id[r + 3] : y0;
        tma_gather4(ring + buf * buf_bytes + qd * quad_stride, &tp.map[cur.k], bar, 0, y0, y1,
                    y2, y3);
      }
    }
    if (cur.valid) advance(bp);
  }

  __device__ __forceinline__ void combine(float (&a)[VEC], const uint4& raw, float w,
                                          bool first) {
    float x[VEC];
    if constexpr (ESZ == 4) {
      x[0] = __uint_as_float(raw.x);
      x[1] = __uint_as_float(raw.y);
      x[2] = __uint_as_float(raw.z);
      x[3] = __uint_as_float(raw.w);
    } else {
      const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        x[2 * e] = __uint_as_float(wv[e] << 16);
        x[2 * e + 1] = __uint_as_float(wv[e] & 0xffff0000u);
      }
    }
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      if (POOL == kPoolSum) {
        a[e] = __fadd_rn(a[e], x[e]);
      } else if (POOL == kPoolWeighted) {
        a[e] = __fmaf_rn(w, x[e], a[e]);
      } else {
        a[e] = first ? x[e] : ((x[e] > a[e]) ? x[e] : a[e]);
      }
    }
  }

  // Consume the next buffer if it belongs to tile `lt` (fused) or exists
  // (gather); refills the previously consumed buffer first. Returns false at
  // the end of the tile or of the sequence. A finished bag's pooled vector
  // goes to `store(meta, chunk m, values)` for each chunk the lane owns.
  template <class Store>
  __device__ __forceinline__ bool step(int lt, const TmaParams& tp, const BagParams& bp,
                                       Store&& store) {
    const int buf = c % kTmaBufs;
    const SegMeta m = meta[buf];
    if (!m.valid || (FUSED && m.lt != lt)) return false;
    issue((c + kTmaBufs - 1) % kTmaBufs, tp, bp);
    if (m.nrows > 0) {
      // after one wait has run out the unit stops waiting: its results are
      // already flagged invalid, and the kernel must still finish promptly
      if (!timeout && !mbar_wait_bounded(bars + buf, (phase >> buf) & 1u, kTmaWaitLimit))
        timeout = true;
      phase ^= 1u << buf;
    }
    if (m.r0 == 0) {
#pragma unroll
      for (int mm = 0; mm < CPL; ++mm)
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[mm][e] = 0.f;
      used = 0;
    }
    const int rows_k = bp.check ? tp.rows[m.k] : 0;
    const unsigned char* base = ring + buf * buf_bytes + q * 16;
    for (int r = 0; r < m.nrows; ++r) {
      const int id = ids[buf * kTmaSegRows + r];
      bool ok = true;
      if (bp.check) {
        ok = static_cast<unsigned>(id) < static_cast<unsigned>(rows_k);
        oob |= !ok;
      }
      if (ok) {
        const float w = POOL == kPoolWeighted ? wts[buf * kTmaSegRows + r] : 0.f;
        const unsigned char* row = base + (r >> 2) * quad_stride + (r & 3) * box_bytes;
#pragma unroll
        for (int mm = 0; mm < CPL; ++mm) {
          if (chunk_ok(mm)) {
            const uint4 raw = *reinterpret_cast<const uint4*>(row + mm * G * 16);
            combine(acc[mm], raw, w, used == 0);
          }
        }
        ++used;
      }
    }
    if (m.r0 + kTmaSegRows >= m.n) {
      if (bp.mean && used > 0) {
        const float cnt = static_cast<float>(used);
#pragma unroll
        for (int mm = 0; mm < CPL; ++mm)
#pragma unroll
          for (int e = 0; e < VEC; ++e) acc[mm][e] = __fdiv_rn(acc[mm][e], cnt);
      }
#pragma unroll
      for (int mm = 0; mm < CPL; ++mm)
        if (chunk_ok(mm)) store(m, mm, acc[mm]);
    }
    __syncwarp(mask);
    fence_proxy_async_smem();  // our reads of this buffer precede its next TMA fill
    ++c;
    return true;
  }
};

// Shared set-up of the gather units of a block.
template <int G, int CPL, int POOL, int ESZ, bool FUSED>
__device__ __forceinline__ void init_unit(TmaUnit<G, CPL, POOL, ESZ, FUSED>& U,
                                          unsigned char* smem, const TmaSmem& L, int B, int F,
                                          int S, int my_tiles) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = warp * (32 / G) + lane / G;
  U.q = lane % G;
  U.mask = (G == 32) ? 0xffffffffu : (((1u << G) - 1u) << (lane - U.q));
  U.ring = smem + static_cast<int64_t>(u) * kTmaBufs * L.buf_bytes;
  U.bars = reinterpret_cast<uint64_t*>(smem + L.bars_off) + u * kTmaBufs;
  U.meta = reinterpret_cast<SegMeta*>(smem + L.meta_off) + u * kTmaBufs;
  U.ids = reinterpret_cast<int32_t*>(smem + L.ids_off) + u * kTmaBufs * kTmaSegRows;
  U.wts = reinterpret_cast<float*>(smem + L.wts_off) + u * kTmaBufs * kTmaSegRows;
  U.buf_bytes = L.buf_bytes;
  U.quad_stride = L.quad_stride;
  U.box_bytes = L.box_bytes;
  U.order = BagOrder<FUSED>{B, F, S, L.units, u, my_tiles};
}

__device__ __forceinline__ void tma_report(const BagParams& bp, bool oob, bool bad, bool tmo) {
  if (bp.status != nullptr) {
    const int flags = (oob ? DLRM_FLAG_INDEX_OOB : 0) | (bad ? DLRM_FLAG_OFFSETS : 0) |
                      (tmo ? DLRM_FLAG_TIMEOUT : 0);
    if (flags) atomicOr(bp.status, flags);
  }
}

// --------------------------------------------------------------------------
// Gather only: persistent blocks of gather units writing pooled rows to `out`.
template <int G, int CPL, int POOL, int ESZ>
__global__ void __launch_bounds__(kTmaGatherWarps * 32, 1)
    tma_embbag_kernel(const __grid_constant__ TmaParams tp, const BagParams bp, int B, int F,
                      int D, float* __restrict__ out) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int VEC = 16 / ESZ;
  const TmaSmem L = TmaSmem::make(G, D * ESZ, 0);
  for (int i = threadIdx.x; i < L.units * kTmaBufs; i += blockDim.x) {
    mbar_init(reinterpret_cast<uint64_t*>(smem + L.bars_off) + i, 1);
  }
  mbar_init_fence();
  __syncthreads();

  TmaUnit<G, CPL, POOL, ESZ, false> U;
  init_unit(U, smem, L, B, F, 1, 0);
  U.start(bp);
  for (int i = 0; i < kTmaBufs - 1; ++i) U.issue(i, tp, bp);
  auto store = [&](const SegMeta& m, int mm, const float (&a)[VEC]) {
    store_vec_f32<VEC>(out + (static_cast<int64_t>(m.b) * F + m.k) * D + (U.q + G * mm) * VEC,
                       a);
  };
  while (U.step(0, tp, bp, store)) {
  }
  if (U.q == 0) tma_report(bp, U.oob, U.bad, U.timeout);
}

// --------------------------------------------------------------------------
// Fused: gather warps pool tile lt into feature buffer lt&1 while dot warps
// finish tile lt-1; each tile holds S consecutive samples.
template <int G, int CPL, int POOL, int ESZ>
__global__ void __launch_bounds__((kTmaGatherWarps + kTmaDotWarps) * 32, 1)
    tma_fused_kernel(const __grid_constant__ TmaParams tp, const BagParams bp,
                     const float* __restrict__ dense, int B, int F, int D, int S, int lq,
                     float* __restrict__ pooled_out, float* __restrict__ inter_out,
                     int concat_dense) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int NT = (kTmaGatherWarps + kTmaDotWarps) * 32;
  constexpr int VEC = 16 / ESZ;
  const FeatLayout Lf = FeatLayout::make(F, D);
  const int64_t sample_floats = Lf.floats_per_sample();
  const TmaSmem L = TmaSmem::make(G, D * ESZ, 2 * S * sample_floats * 4);
  float* feat = reinterpret_cast<float*>(smem + L.feat_off);
  const int64_t ntiles = (static_cast<int64_t>(B) + S - 1) / S;
  const int my_tiles = blockIdx.x < ntiles
                           ? static_cast<int>((ntiles - 1 - blockIdx.x) / gridDim.x + 1)
                           : 0;
  for (int i = threadIdx.x; i < L.units * kTmaBufs; i += blockDim.x) {
    mbar_init(reinterpret_cast<uint64_t*>(smem + L.bars_off) + i, 1);
  }
  mbar_init_fence();
  __syncthreads();

  const int64_t P = static_cast<int64_t>(Lf.F1) * (Lf.F1 - 1) / 2;
  const int64_t row_stride = concat_dense ? D + P : P;
  const int warp = threadIdx.x >> 5;

  if (warp < kTmaGatherWarps) {
    TmaUnit<G, CPL, POOL, ESZ, true> U;
    init_unit(U, smem, L, B, F, S, my_tiles);
    U.start(bp);
    for (int i = 0; i < kTmaBufs - 1; ++i) U.issue(i, tp, bp);
    for (int lt = 0; lt < my_tiles; ++lt) {
      const int p = lt & 1;
      if (lt >= 2) named_bar_sync(kBarFree0 + p, NT);
      float* fb = feat + p * S * sample_floats;
      const int64_t b0 = (static_cast<int64_t>(blockIdx.x) + static_cast<int64_t>(lt) *
                                                                 gridDim.x) * S;
      auto store = [&](const SegMeta& m, int mm, const float (&a)[VEC]) {
        const int s = static_cast<int>(m.b - b0);
        const int col = (U.q + G * mm) * VEC;
        store_vec_f32<VEC>(fb + s * sample_floats + (1 + m.k) * Lf.Dp + col, a);
        if (pooled_out)
          store_vec_f32<VEC>(pooled_out + (static_cast<int64_t>(m.b) * F + m.k) * D + col, a);
      };
      while (U.step(lt, tp, bp, store)) {
      }
      __syncwarp();
      named_bar_arrive(kBarReady0 + p, NT);
    }
    if (U.q == 0) tma_report(bp, U.oob, U.bad, U.timeout);
  } else {
    fused_dot_warps<kTmaGatherWarps, kTmaDotWarps>(feat, Lf, dense, B, D, S, lq, my_tiles,
                                                   inter_out, concat_dense);
  }
}

// --------------------------------------------------------------------------
// Host-side dispatch.

template <int G, int CPL, int POOL, int ESZ>
cudaError_t run_tma_gather(const TmaLaunch& a) {
  auto* fn = &tma_embbag_kernel<G, CPL, POOL, ESZ>;
  const TmaSmem L = TmaSmem::make(G, a.D * ESZ, 0);
  cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(fn),
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(L.total));
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kTmaGatherWarps * 32, L.total);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int64_t work = (static_cast<int64_t>(a.B) * a.F + L.units - 1) / L.units;
  const int64_t grid = std::min<int64_t>(static_cast<int64_t>(per_sm) * a.sms, work);
  fn<<<static_cast<unsigned>(grid), kTmaGatherWarps * 32, L.total, a.stream>>>(*a.tp, a.bp, a.B,
                                                                                a.F, a.D, a.out);
  return cudaGetLastError();
}

template <int G, int CPL, int POOL, int ESZ>
cudaError_t run_tma_fused(const TmaLaunch& a) {
  auto* fn = &tma_fused_kernel<G, CPL, POOL, ESZ>;
  const FeatLayout Lf = FeatLayout::make(a.F, a.D);
  const TmaSmem L = TmaSmem::make(G, a.D * ESZ, 2 * a.S * Lf.floats_per_sample() * 4);
  if (L.total > a.smem_limit) return cudaErrorInvalidValue;
  constexpr int NT = (kTmaGatherWarps + kTmaDotWarps) * 32;
  cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(fn),
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(L.total));
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, NT, L.total);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int64_t ntiles = (static_cast<int64_t>(a.B) + a.S - 1) / a.S;
  const int64_t grid = std::min<int64_t>(static_cast<int64_t>(per_sm) * a.sms, ntiles);
  fn<<<static_cast<unsigned>(grid), NT, L.total, a.stream>>>(
      *a.tp, a.bp, a.dense, a.B, a.F, a.D, a.S, a.lq, a.pooled_out, a.inter_out, a.concat_dense);
  return cudaGetLastError();
}

// Lanes per unit and 16-byte chunks per lane for a row of `row_bytes`:
// G = 8 (32 units per block) up to 256-byte rows, G = 16 (16 units) above.
__host__ __device__ inline int tma_unit_lanes(int row_bytes) { return row_bytes <= 256 ? 8 : 16; }
__host__ __device__ inline int tma_chunks_per_lane(int row_bytes) {
  const int G = tma_unit_lanes(row_bytes);
  return (row_bytes / 16 + G - 1) / G;
}

#define DLRM_TMA_POOLS(RUN, G_, C_, ESZ_, a)                                      \
  do {                                                                          \
    if ((a).pool == kPoolSum) return RUN<G_, C_, kPoolSum, ESZ_>(a);            \
    if ((a).pool == kPoolWeighted) return RUN<G_, C_, kPoolWeighted, ESZ_>(a);  \
    return RUN<G_, C_, kPoolMax, ESZ_>(a);                                      \
  } while (0)

#define DLRM_TMA_DISPATCH(RUN, ESZ_, a)                                          \
  do {                                                                          \
    if ((a).G == 8 && (a).cpl == 1) DLRM_TMA_POOLS(RUN, 8, 1, ESZ_, a);          \
    if ((a).G == 8) DLRM_TMA_POOLS(RUN, 8, 2, ESZ_, a);                         \
    DLRM_TMA_POOLS(RUN, 16, 2, ESZ_, a);                                        \
  } while (0)

}  // namespace dlrm
