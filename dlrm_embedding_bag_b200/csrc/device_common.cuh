// Device-side building blocks shared by the gather, interaction and fused
// kernels of the DLRMv1 sparse/interaction stage (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "dlrm_sparse.h"

namespace dlrm {

constexpr unsigned kFullMask = 0xffffffffu;
// Threads of a gather, fused or interaction block. Measured on B200 against
// 256-thread blocks (eight blocks per SM instead of four, same 64 registers):
// fused c3 49.7 -> 48.8 us, c2 33.4 -> 32.5 us, c5 1.60 -> 1.56 ms, bf16 tables
// 44.0 -> 41.9 us, the interaction alone at c3 20.8 -> 18.9 us; c3u the same.
// More, smaller blocks overlap one block's barrier and dot phase with other
// blocks' gathers.
constexpr int kBlockThreads = 128;

// The F table base pointers (and, for the checked entry points, their row
// counts) travel by value in the kernel's parameter block (__grid_constant__),
// so a launch needs no device-side pointer array and no host-to-device copy.
struct TableParams {
  const void* w[DLRM_MAX_TABLES];
  int32_t rows[DLRM_MAX_TABLES];
};

// Where the bags are and how they pool.
struct BagParams {
  const int32_t* indices;  // (F, T) table-major
  const int32_t* offsets;  // (F, B) or (F, B + 1) with include_last_offset
  const float* psw;        // (F, T) per-sample weights, or null
  int T;                   // index entries per table
  int ilo;                 // include_last_offset
  int mean;                // divide each pooled sum by the bag's entry count
  int check;               // skip (and flag) indices outside [0, rows[k])
  int32_t* status;         // device flags, or null
  int balance;             // fused kernel: order each block's bags by length
};

// Pooling combine step, fixed per template instance.
enum PoolKind { kPoolSum = 0, kPoolWeighted = 1, kPoolMax = 2 };

// ---------------------------------------------------------------------------
// Row loaders: one lane loads VEC consecutive table elements per request and
// hands them out widened to f32.

// Row loads that do not allocate in L1 (ld.global.nc.L1::no_allocate), for
// rows that are read once per lookup and rarely again by the same SM: L1 is
// left to the requests in flight. Measured on B200 against plain __ldg, with
// 256-byte f32 rows (D = 64): fused c3 52.2 -> 49.9 us, c3u 70.1 -> 66.0 us,
// gather alone c3u 65.0 -> 58.6 us; but with 512-byte rows under a steeper
// skew (c5: D = 128, Zipf 1.2) 1.62 -> 1.70 ms and with 128-byte bf16 rows
// 44.6 -> 49.0 us, where L1 serves enough hot rows to pay. So the launch picks
// the streaming loader (LdF32x4S) for f32 rows of at most 64 floats only.
__device__ __forceinline__ float4 ldg_row_f32x4(const float* p) {
  float4 r;
  asm("ld.global.nc.L1::no_allocate.v4.f32 {%0, %1, %2, %3}, [%4];"
      : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
      : "l"(p));
  return r;
}
struct LdF32x4 {  // 128-bit loads of 4 floats
  static constexpr int VEC = 4;
  using Elem = float;
  using Raw = float4;
  __device__ __forceinline__ static Raw zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ __forceinline__ static Raw load(const Elem* p) {
    return __ldg(reinterpret_cast<const float4*>(p));
  }
  __device__ __forceinline__ static float get(const Raw& r, int e) {
    return e == 0 ? r.x : e == 1 ? r.y : e == 2 ? r.z : r.w;
  }
};

struct LdF32x4S : LdF32x4 {  // the same, streaming (no L1 allocation)
  __device__ __forceinline__ static Raw load(const Elem* p) { return ldg_row_f32x4(p); }
};

struct LdF32x1 {  // scalar fallback
  static constexpr int VEC = 1;
  using Elem = float;
  using Raw = float;
  __device__ __forceinline__ static Raw zero() { return 0.f; }
  __device__ __forceinline__ static Raw load(const Elem* p) { return __ldg(p); }
  __device__ __forceinline__ static float get(const Raw& r, int) { return r; }
};

// A bf16 value is the upper half of an f32: widening is a 16-bit shift.
__device__ __forceinline__ float bf16_bits_to_float(uint32_t h16) {
  return __uint_as_float(h16 << 16);
}

struct LdBF16x8 {  // 128-bit loads of 8 bf16
  static constexpr int VEC = 8;
  using Elem = uint16_t;
  using Raw = uint4;
  __device__ __forceinline__ static Raw zero() { return make_uint4(0u, 0u, 0u, 0u); }
  __device__ __forceinline__ static Raw load(const Elem* p) {
    return __ldg(reinterpret_cast<const uint4*>(p));
  }
  __device__ __forceinline__ static float get(const Raw& r, int e) {
    const uint32_t w = (e >> 1) == 0 ? r.x : (e >> 1) == 1 ? r.y : (e >> 1) == 2 ? r.z : r.w;
    return (e & 1) ? __uint_as_float(w & 0xffff0000u) : __uint_as_float(w << 16);
  }
};

struct LdBF16x1 {  // scalar fallback
  static constexpr int VEC = 1;
  using Elem = uint16_t;
  using Raw = unsigned short;
  __device__ __forceinline__ static Raw zero() { return 0; }
  __device__ __forceinline__ static Raw load(const Elem* p) {
    return __ldg(reinterpret_cast<const unsigned short*>(p));
  }
  __device__ __forceinline__ static float get(const Raw& r, int) {
    return bf16_bits_to_float(static_cast<uint32_t>(r));
  }
};

// Flat index p of the strict lower triangle (row-major, i > j) -> (i, j):
// i = floor((1 + sqrt(1 + 8p)) / 2), j = p - i(i-1)/2. The square root is
// taken in f32 and the integer correction afterwards makes
// i(i-1)/2 <= p < i(i+1)/2 hold exactly; each correction loop moves i
// monotonically toward that unique value, so both terminate.
__device__ __forceinline__ void pair_from_flat(int64_t p, int& i_out, int& j_out) {
  float t = sqrtf(8.0f * static_cast<float>(p) + 1.0f);
  int64_t i = static_cast<int64_t>((t + 1.0f) * 0.5f);
  if (i < 1) i = 1;
  while (i * (i - 1) / 2 > p) --i;
  while (i * (i + 1) / 2 <= p) ++i;
  i_out = static_cast<int>(i);
  j_out = static_cast<int>(p - i * (i - 1) / 2);
}

// The same decoder for small p (< 2^24, where every int is exact in f32); the
// interaction's dot phase decodes its tile index with it.
constexpr int64_t kPairSmallLimit = int64_t{1} << 24;
__device__ __forceinline__ void pair_from_flat_small(int p, int& i_out, int& j_out) {
  int i = static_cast<int>((sqrtf(8.0f * static_cast<float>(p) + 1.0f) + 1.0f) * 0.5f);
  if (i < 1) i = 1;
  while (i * (i - 1) / 2 > p) --i;
  while (i * (i + 1) / 2 <= p) ++i;
  i_out = i;
  j_out = p - i * (i - 1) / 2;
}

// Bag bounds of (table k, sample b) under torch's offsets rule: the bag ends
// where the next one starts, or at T for the last bag (include_last_offset=0),
// or at offsets[k][B] (include_last_offset=1). Invalid bounds give an empty
// bag and raise *bad.
// Sort keys of the fused kernel's bag ordering: (length + 1) << 11 | bag.
constexpr int kSortTaskBits = 11;  // bags per block < 2048
constexpr int kSortLenMax = (1 << (32 - kSortTaskBits)) - 2;

// Sorts one key per lane across the warp, largest at lane 0: Batcher's
// bitonic network, log2(32) merge phases of shuffle-exchange steps. In phase
// k the runs of k lanes alternate direction so that each pair of runs forms a
// bitonic sequence for the next phase; the last phase runs one direction.
__device__ __forceinline__ unsigned warp_sort_desc(unsigned key, int lane) {
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const unsigned other = __shfl_xor_sync(kFullMask, key, j);
      const bool keep_max = ((lane & j) == 0) == ((lane & k) == 0);
      key = keep_max ? max(key, other) : min(key, other);
    }
  }
  return key;
}

__device__ __forceinline__ void bag_bounds(const BagParams& bp, int B, int k, int b, int& start,
                                           int& n, bool& bad) {
  const int64_t o = static_cast<int64_t>(k) * (B + bp.ilo) + b;
  const int s = __ldg(bp.offsets + o);
  const int e = (bp.ilo || b + 1 < B) ? __ldg(bp.offsets + o + 1) : bp.T;
  bad = (s < 0) || (s > e) || (e > bp.T);
  start = bad ? 0 : s;
  n = bad ? 0 : e - s;
}

// Pool one bag for the columns this lane owns; returns the entries used.
//
// A lane group of G consecutive lanes handles one bag; lane q owns the column
// chunks q, q+G, ..., q+(CPL-1)G of the current column window (a chunk is VEC
// consecutive elements). Rows are fetched U at a time, all U loads issued
// before any is consumed; the bag's row ids (and weights) are read once,
// coalesced, by the group and handed out with warp shuffles. Each column then
// combines the rows in bag order with one rounding per step (an add, a fused
// multiply-add, or a comparison), so the result is bit-identical to the
// sequential definition.
//
// Every lane of the warp must call this with the same `nmax` (the largest n in
// the warp), because the shuffles run over the full warp.
template <class LD, int G, int CPL, int U, int POOL>
__device__ __forceinline__ int pool_bag(const typename LD::Elem* __restrict__ W, int rows_k,
                                        bool check, const int32_t* __restrict__ idx_seg,
                                        const float* __restrict__ w_seg, int start, int n,
                                        int nmax, int D, int col0, int q, int gbase,
                                        float (&acc)[CPL][LD::VEC], bool& oob) {
  constexpr int VEC = LD::VEC;
  // Row ids are fetched NB at a time (one coalesced load per lane), rows U at
  // a time out of those, so a bag of up to NB rows costs one id round trip.
  constexpr int NB = U > G ? U : G;
  constexpr int IPL = NB / G;  // row ids held per lane
#pragma unroll
  for (int m = 0; m < CPL; ++m)
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[m][e] = 0.f;
  bool colok[CPL];
  bool all_cols = true;
#pragma unroll
  for (int m = 0; m < CPL; ++m) {
    colok[m] = col0 + (q + G * m) * VEC < D;
    all_cols = all_cols && colok[m];
  }
  // Batches that every bag of the warp covers entirely, with every column
  // chunk in range and no index check, take a path with no predicates (for
  // max pooling, `have` is the same in every lane of such a batch: all bags of
  // the warp have had the same number of entries combined so far).
  const bool plain = !check && __all_sync(kFullMask, all_cols);
  int used = 0;       // entries used; counted only under `check` (else every entry is)
  bool have = false;  // max pooling: an entry has been combined

  for (int c = 0; c < nmax; c += NB) {
    int my_row[IPL];
    float my_w[IPL];
#pragma unroll
    for (int j = 0; j < IPL; ++j) {
      const int t = c + q + G * j;
      const bool in = t < n;
      my_row[j] = in ? __ldg(idx_seg + start + t) : 0;
      if (POOL == kPoolWeighted) my_w[j] = in ? __ldg(w_seg + start + t) : 0.f;
    }
#pragma unroll
    for (int cu = 0; cu < NB; cu += U) {
      if (c + cu >= nmax) break;  // warp-uniform
      // Weights are handed out at combine time (not with the row loads), so
      // U of them need not stay live across the loads.
      typename LD::Raw v[U][CPL];
      if (plain && __all_sync(kFullMask, c + cu + U <= n)) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int slot = cu + u;
          const int r = __shfl_sync(kFullMask, my_row[slot / G], gbase + (slot % G));
          const typename LD::Elem* row = W + static_cast<int64_t>(r) * D + col0 + q * VEC;
#pragma unroll
          for (int m = 0; m < CPL; ++m) v[u][m] = LD::load(row + G * m * VEC);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int slot = cu + u;
          float wt = 0.f;
          if (POOL == kPoolWeighted)
            wt = __shfl_sync(kFullMask, my_w[slot / G], gbase + (slot % G));
#pragma unroll
          for (int m = 0; m < CPL; ++m)
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
              const float x = LD::get(v[u][m], e);
              if constexpr (POOL == kPoolMax) {
                // the bag's first entry starts the maximum (warp-uniform test)
                acc[m][e] = (u == 0 && !have) ? x : ((x > acc[m][e]) ? x : acc[m][e]);
              } else {
                acc[m][e] = (POOL == kPoolSum) ? __fadd_rn(acc[m][e], x)
                                               : __fmaf_rn(wt, x, acc[m][e]);
              }
            }
        }
        have = true;
        continue;
      }
      bool use[U];  // entry cu + u is combined
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int slot = cu + u;
        const int r = __shfl_sync(kFullMask, my_row[slot / G], gbase + (slot % G));
        bool ok = (c + slot) < n;
        if (check) {
          const bool in_range = static_cast<unsigned>(r) < static_cast<unsigned>(rows_k);
          oob |= ok && !in_range;
          ok = ok && in_range;
          used += ok ? 1 : 0;
        }
        use[u] = ok;
        const typename LD::Elem* row = W + static_cast<int64_t>(r) * D + col0 + q * VEC;
#pragma unroll
        for (int m = 0; m < CPL; ++m) {
          v[u][m] = LD::zero();
          if (ok && colok[m]) v[u][m] = LD::load(row + G * m * VEC);
        }
      }
      if (POOL != kPoolMax) {
        // A skipped entry adds +0.0 (weight 0 times 0): the running sum starts
        // at +0.0 and never becomes -0.0 under round-to-nearest, so adding +0.0
        // leaves it unchanged, bit for bit, and no branch is needed.
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int slot = cu + u;
          float wt = 0.f;
          if (POOL == kPoolWeighted) {
            wt = __shfl_sync(kFullMask, my_w[slot / G], gbase + (slot % G));
            wt = use[u] ? wt : 0.f;
          }
#pragma unroll
          for (int m = 0; m < CPL; ++m)
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
              const float x = LD::get(v[u][m], e);
              acc[m][e] = (POOL == kPoolSum) ? __fadd_rn(acc[m][e], x)
                                             : __fmaf_rn(wt, x, acc[m][e]);
            }
        }
      } else {
#pragma unroll
        for (int u = 0; u < U; ++u) {
          if (use[u]) {
#pragma unroll
            for (int m = 0; m < CPL; ++m)
#pragma unroll
              for (int e = 0; e < VEC; ++e) {
                const float x = LD::get(v[u][m], e);
                acc[m][e] = have ? ((x > acc[m][e]) ? x : acc[m][e]) : x;
              }
            have = true;
          }
        }
      }
    }
  }
  return check ? used : n;
}

// Mean pooling: one division of the sequential sum by the entries used.
template <int CPL, int VEC>
__device__ __forceinline__ void finish_mean(float (&acc)[CPL][VEC], int used) {
  if (used > 0) {
    const float cnt = static_cast<float>(used);
#pragma unroll
    for (int m = 0; m < CPL; ++m)
#pragma unroll
      for (int e = 0; e < VEC; ++e) acc[m][e] = __fdiv_rn(acc[m][e], cnt);
  }
}

// Store VEC consecutive floats (16-byte aligned when VEC is 4 or 8).
template <int VEC>
__device__ __forceinline__ void store_floats(float* p, const float (&a)[VEC]) {
  if constexpr (VEC % 4 == 0) {
#pragma unroll
    for (int e = 0; e < VEC; e += 4)
      *reinterpret_cast<float4*>(p + e) = make_float4(a[e], a[e + 1], a[e + 2], a[e + 3]);
  } else {
#pragma unroll
    for (int e = 0; e < VEC; ++e) p[e] = a[e];
  }
}

}  // namespace dlrm
