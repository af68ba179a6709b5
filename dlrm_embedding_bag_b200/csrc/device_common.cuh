// Device-side building blocks shared by the gather, interaction and fused
// kernels of the DLRMv1 sparse/interaction stage (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "dlrm_sparse.h"

namespace dlrm {

constexpr unsigned kFullMask = 0xffffffffu;
constexpr int kBlockThreads = 256;

// The F table base pointers (and, for the checked entry points, their row
// counts) travel by value in the kernel's parameter block (__grid_constant__),
// so a launch needs no device-side pointer array and no host-to-device copy.
struct TableParams {
  const float* w[DLRM_MAX_TABLES];
  int32_t rows[DLRM_MAX_TABLES];
};

// 128-bit and 32-bit read-only loads of table rows.
__device__ __forceinline__ float4 load_row_chunk(const float* p, float4*) {
  return __ldg(reinterpret_cast<const float4*>(p));
}
__device__ __forceinline__ float load_row_chunk(const float* p, float*) { return __ldg(p); }

__device__ __forceinline__ void acc_add(float4& a, const float4& v) {
  a.x = __fadd_rn(a.x, v.x);
  a.y = __fadd_rn(a.y, v.y);
  a.z = __fadd_rn(a.z, v.z);
  a.w = __fadd_rn(a.w, v.w);
}
__device__ __forceinline__ void acc_add(float& a, const float& v) { a = __fadd_rn(a, v); }

__device__ __forceinline__ void set_zero(float4& a) { a = make_float4(0.f, 0.f, 0.f, 0.f); }
__device__ __forceinline__ void set_zero(float& a) { a = 0.f; }

template <int VEC>
struct VecOf;
template <>
struct VecOf<4> {
  using T = float4;
};
template <>
struct VecOf<1> {
  using T = float;
};

__device__ __forceinline__ void store_vec(float* p, const float4& v) {
  *reinterpret_cast<float4*>(p) = v;
}
__device__ __forceinline__ void store_vec(float* p, const float& v) { *p = v; }

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

// Bag bounds of (table k, sample b) under the include_last_offset=False rule.
// Invalid offsets give an empty bag and raise *bad.
__device__ __forceinline__ void bag_bounds(const int32_t* __restrict__ offsets, int B, int BL,
                                           int k, int b, int& start, int& n, bool& bad) {
  const int64_t o = static_cast<int64_t>(k) * B + b;
  const int s = __ldg(offsets + o);
  const int e = (b + 1 < B) ? __ldg(offsets + o + 1) : BL;
  bad = (s < 0) || (s > e) || (e > BL);
  start = bad ? 0 : s;
  n = bad ? 0 : e - s;
}

// Pool one bag for the columns this lane owns.
//
// A lane group of G consecutive lanes handles one bag; lane q owns the column
// chunks q, q+G, ..., q+(CPL-1)G of the current column window (a chunk is VEC
// consecutive floats). Rows are fetched U at a time, all U loads issued before
// any is consumed; the bag's row ids are read once, coalesced, by the group
// and handed out with warp shuffles. Each column is then accumulated from
// 0.0f in bag order with one rounding per add, so the result is bit-identical
// to the sequential f32 sum.
//
// Every lane of the warp must call this with the same `nmax` (the largest n in
// the warp), because the shuffles run over the full warp.
template <int VEC, int G, int CPL, int U, bool CHECK>
__device__ __forceinline__ void pool_bag(const float* __restrict__ W, int rows_k,
                                         const int32_t* __restrict__ idx_seg, int start, int n,
                                         int nmax, int D, int col0, int q, int gbase,
                                         typename VecOf<VEC>::T (&acc)[CPL], bool& oob) {
  using V = typename VecOf<VEC>::T;
  constexpr int IPL = (U + G - 1) / G;  // row ids held per lane per batch of U rows
#pragma unroll
  for (int m = 0; m < CPL; ++m) set_zero(acc[m]);

  for (int c = 0; c < nmax; c += U) {
    int my_row[IPL];
#pragma unroll
    for (int j = 0; j < IPL; ++j) {
      const int slot = q + G * j;
      const int t = c + slot;
      my_row[j] = (slot < U && t < n) ? __ldg(idx_seg + start + t) : 0;
    }
    V v[U][CPL];
    bool use[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int r = __shfl_sync(kFullMask, my_row[u / G], gbase + (u % G));
      bool ok = (c + u) < n;
      if (CHECK) {
        const bool in_range = (r >= 0) && (r < rows_k);
        oob |= ok && !in_range;
        ok = ok && in_range;
      }
      use[u] = ok;
      const float* row = W + static_cast<int64_t>(r) * D;
#pragma unroll
      for (int m = 0; m < CPL; ++m) {
        const int col = col0 + (q + G * m) * VEC;
        if (ok && col < D) {
          v[u][m] = load_row_chunk(row + col, static_cast<V*>(nullptr));
        } else {
          set_zero(v[u][m]);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (use[u]) {
#pragma unroll
        for (int m = 0; m < CPL; ++m) acc_add(acc[m], v[u][m]);
      }
    }
  }
}

}  // namespace dlrm
