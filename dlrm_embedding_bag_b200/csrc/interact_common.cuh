// Shared-memory pairwise-dot phase of the interaction (sm_100a).
#pragma once

#include "device_common.cuh"

namespace dlrm {

// Shared-memory feature block of one sample: F1p = 4*ceil((F+1)/4) rows (dense
// first, then the F pooled vectors, then up to 3 filler rows), each
// Dp = 4*ceil(D/4) + 4 floats long. The row length keeps every row 16-byte
// aligned for float4 reads, and the extra 4 floats shift consecutive rows by
// one 16-byte bank group, so float4 reads of different rows at the same
// column do not collide.
struct FeatLayout {
  int F1;   // features = F + 1
  int F1p;  // rows per sample, multiple of 4
  int D4;   // float4 chunks per row holding data (ceil(D/4))
  int Dp;   // floats per row
  int nT;   // 4x4 pair tiles of the lower triangle incl. the diagonal tiles
  __host__ __device__ static FeatLayout make(int F, int D) {
    FeatLayout L;
    L.F1 = F + 1;
    L.F1p = 4 * ((L.F1 + 3) / 4);
    L.D4 = (D + 3) / 4;
    L.Dp = 4 * L.D4 + 4;
    const int nI = L.F1p / 4;
    L.nT = nI * (nI + 1) / 2;
    return L;
  }
  __host__ __device__ int64_t floats_per_sample() const {
    return static_cast<int64_t>(F1p) * Dp;
  }
};

// Zero what the dot phase reads but the loaders do not write: the columns
// [D, 4*D4) of the feature rows, and the filler rows [F1, F1p). (The filler
// rows only feed tile entries that are never stored; they are zeroed so that
// nothing reads uninitialised memory.)
//
// Run by the `nthreads` threads tid = 0 .. nthreads-1 (a multiple of 32).
__device__ __forceinline__ void zero_feature_padding(float* feat, const FeatLayout& Lf, int D,
                                                     int S_here, int tid, int nthreads) {
  const int padc = 4 * Lf.D4 - D;  // 0..3
  const int warp = tid >> 5, lane = tid & 31, nwarps = nthreads >> 5;
  for (int s = 0; s < S_here; ++s) {
    float* base = feat + static_cast<int64_t>(s) * Lf.F1p * Lf.Dp;
    if (padc > 0) {
      for (int f = warp; f < Lf.F1; f += nwarps)
        if (lane < padc) base[f * Lf.Dp + D + lane] = 0.f;
    }
    const int n_extra = (Lf.F1p - Lf.F1) * Lf.Dp;
    for (int e = tid; e < n_extra; e += nthreads) base[Lf.F1 * Lf.Dp + e] = 0.f;
  }
}

// All strict-lower-triangle dots of the block's samples, from shared memory.
//
// The pairs are covered by 4x4 tiles (I, J), I >= J, of the (F+1) x (F+1)
// Gram matrix; the flat tile index t is decoded with the same closed form as
// the pair index (tile (I, J) is pair (I+1, J) of a triangle one larger). A
// task is (sample, tile, q): Q = 2^lq consecutive lanes split the D columns
// of one tile (lane q takes float4 chunks q, q+Q, ...), keep the 16 partial
// dots in registers (each float4 read from shared memory feeds 16 FMAs), and
// combine them with xor shuffles. Lane q then stores the tile entries
// e = 4r + c with e % Q == q that lie strictly below the diagonal and inside
// F+1.
//
// The output row of sample b starts at out + b * row_stride + col0; dot p of
// the row is written at offset p. Run by the `nthreads` threads tid = 0 ..
// nthreads-1 (a multiple of 32, whole warps).
__device__ __forceinline__ void dots_from_smem(const float* feat, const FeatLayout& Lf,
                                               int S_here, int lq, float* __restrict__ out,
                                               int64_t b0, int64_t row_stride, int64_t col0,
                                               int tid, int nthreads) {
  const int Q = 1 << lq;
  const int total = (S_here * Lf.nT) << lq;
  const int lane = tid & 31;
  for (int base = tid - lane; base < total; base += nthreads) {
    const int task = base + lane;
    const bool active = task < total;
    const int tt = active ? task : 0;
    const int q = tt & (Q - 1);
    const int rest = tt >> lq;
    int t = rest, s = 0;
    if (S_here > 1) {
      s = rest / Lf.nT;
      t = rest - s * Lf.nT;
    }
    int I1, J;
    pair_from_flat_small(t, I1, J);
    const int I = I1 - 1;
    const float* fi = feat + (static_cast<int64_t>(s) * Lf.F1p + 4 * I) * Lf.Dp;
    const float* fj = feat + (static_cast<int64_t>(s) * Lf.F1p + 4 * J) * Lf.Dp;

    float acc[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;

    for (int d4 = q; d4 < Lf.D4; d4 += Q) {
      float4 a[4], bv[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) a[r] = *reinterpret_cast<const float4*>(fi + r * Lf.Dp + 4 * d4);
#pragma unroll
      for (int c = 0; c < 4; ++c) bv[c] = *reinterpret_cast<const float4*>(fj + c * Lf.Dp + 4 * d4);
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float x = acc[r][c];
          x = fmaf(a[r].x, bv[c].x, x);
          x = fmaf(a[r].y, bv[c].y, x);
          x = fmaf(a[r].z, bv[c].z, x);
          x = fmaf(a[r].w, bv[c].w, x);
          acc[r][c] = x;
        }
    }
    for (int off = 1; off < Q; off <<= 1) {
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] += __shfl_xor_sync(kFullMask, acc[r][c], off);
    }
    if (active) {
      float* orow = out + (b0 + s) * row_stride + col0;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int i = 4 * I + r;
        if (i >= Lf.F1) continue;
        float* orow_i = orow + i * (i - 1) / 2 + 4 * J;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (((4 * r + c) & (Q - 1)) == q && 4 * J + c < i) orow_i[c] = acc[r][c];
        }
      }
    }
  }
}

}  // namespace dlrm
