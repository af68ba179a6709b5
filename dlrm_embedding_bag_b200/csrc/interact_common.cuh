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

// Reduce-scatter of one 4x4 tile of partial dots over the Q = 2^LQ lanes of
// a task, then the stores. Tile value v = 4r + c is the dot of rows 4I+r and
// 4J+c. Each xor round halves what a lane holds: the lane whose mask bit is
// clear keeps the lower half of its values and receives its partner's lower
// half, the other keeps and receives the upper half. After LQ rounds lane q
// holds the fully summed values v = q*(16/Q) .. q*(16/Q) + 16/Q - 1, and
// stores the ones strictly below the diagonal and inside F+1.
template <int LQ>
__device__ __forceinline__ void tile_reduce_store(float (&acc)[16], int q, bool active, int I,
                                                  int J, int F1, float* __restrict__ orow) {
  constexpr int Q = 1 << LQ;
  constexpr int NV = 16 >> LQ;
#pragma unroll
  for (int round = 0; round < LQ; ++round) {
    const int m = Q >> (round + 1);
    const int half = 8 >> round;
    const bool upper = (q & m) != 0;
#pragma unroll
    for (int k = 0; k < half; ++k) {
      const float lo = acc[k], hi = acc[k + half];
      const float send = upper ? lo : hi;
      const float keep = upper ? hi : lo;
      acc[k] = keep + __shfl_xor_sync(kFullMask, send, m);
    }
  }
  if (!active) return;
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int v = q * NV + k;
    const int i = 4 * I + (v >> 2);
    const int j = 4 * J + (v & 3);
    if (i < F1 && j < i) orow[i * (i - 1) / 2 + j] = acc[k];
  }
}

// All strict-lower-triangle dots of the block's samples, from shared memory.
//
// The pairs are covered by 4x4 tiles (I, J), I >= J, of the (F+1) x (F+1)
// Gram matrix; the flat tile index t is decoded with the same closed form as
// the pair index (tile (I, J) is pair (I+1, J) of a triangle one larger). A
// task is (sample, tile, q): Q = 2^lq consecutive lanes (lq <= 4) split the D
// columns of one tile (lane q takes float4 chunks q, q+Q, ...) and keep the 16
// partial dots in registers, so each float4 read from shared memory feeds 16
// FMAs; tile_reduce_store combines and stores them.
//
// The output row of sample b starts at out + b * row_stride + col0; dot p of
// the row is written at offset p. Run by the `nthreads` threads tid = 0 ..
// nthreads-1 (a multiple of 32, whole warps). UNROLL iterations of the column
// loop are unrolled (more loads in flight, more registers). DP > 0 fixes the
// row length Lf.Dp at compile time, so every shared-memory read of a tile
// step is an immediate offset from one of two base addresses.
template <int UNROLL = 1, int DP = 0>
__device__ __forceinline__ void dots_from_smem(const float* feat, const FeatLayout& Lf,
                                               int S_here, int lq, float* __restrict__ out,
                                               int64_t b0, int64_t row_stride, int64_t col0,
                                               int tid, int nthreads) {
  const int Q = 1 << lq;
  const int total = (S_here * Lf.nT) << lq;
  const int lane = tid & 31;
  const int rstride = DP > 0 ? (DP >> 2) : (Lf.Dp >> 2);  // float4 per feature row
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
    const float4* fi = reinterpret_cast<const float4*>(feat) +
                       (static_cast<int64_t>(s) * Lf.F1p + 4 * I) * rstride + q;
    const float4* fj = reinterpret_cast<const float4*>(feat) +
                       (static_cast<int64_t>(s) * Lf.F1p + 4 * J) * rstride + q;

    float acc[16];
#pragma unroll
    for (int v = 0; v < 16; ++v) acc[v] = 0.f;

#pragma unroll UNROLL
    for (int d4 = q; d4 < Lf.D4; d4 += Q) {
      float4 a[4], bv[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) a[r] = fi[r * rstride];
#pragma unroll
      for (int c = 0; c < 4; ++c) bv[c] = fj[c * rstride];
      fi += Q;
      fj += Q;
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float x = acc[4 * r + c];
          x = fmaf(a[r].x, bv[c].x, x);
          x = fmaf(a[r].y, bv[c].y, x);
          x = fmaf(a[r].z, bv[c].z, x);
          x = fmaf(a[r].w, bv[c].w, x);
          acc[4 * r + c] = x;
        }
    }
    float* orow = out + (b0 + s) * row_stride + col0;
    switch (lq) {
      case 0: tile_reduce_store<0>(acc, q, active, I, J, Lf.F1, orow); break;
      case 1: tile_reduce_store<1>(acc, q, active, I, J, Lf.F1, orow); break;
      case 2: tile_reduce_store<2>(acc, q, active, I, J, Lf.F1, orow); break;
      case 3: tile_reduce_store<3>(acc, q, active, I, J, Lf.F1, orow); break;
      default: tile_reduce_store<4>(acc, q, active, I, J, Lf.F1, orow); break;
    }
  }
}

// The 4x4 tiles (I, J), I >= J, of the lower triangle, decoded once per block
// from their flat index with the pair decoder (tile (I, J) is pair (I+1, J) of
// a triangle one larger): tiles[t] = I << 8 | J. Run by nthreads threads.
__device__ __forceinline__ void decode_tiles(uint16_t* tiles, int nT, int tid, int nthreads) {
  for (int t = tid; t < nT; t += nthreads) {
    int I1, J;
    pair_from_flat_small(t, I1, J);
    tiles[t] = static_cast<uint16_t>(((I1 - 1) << 8) | J);
  }
}

// dots_from_smem for a row length fixed at compile time: D4 float4 chunks of
// data per feature row, RS float4 per row in shared memory, 2^LQ lanes per
// tile, tiles from the table decode_tiles wrote. Every shared-memory read of
// a tile is an immediate offset from one of two base addresses and the column
// loop is fully unrolled. Same tasks and stores as dots_from_smem; each dot
// keeps two partial sums (its even and its odd columns) updated by packed
// two-lane FMAs, added once at the end (measured on B200: the interaction at
// B=65536, F=26, D=128 332.5 -> 317.4 us; unchanged at B=2048, F=32, D=64).

// Two round-to-nearest f32 fused multiply-adds in one packed instruction
// (sm_100 fma.rn.f32x2): (d0, d1) = (a0 * b0 + d0, a1 * b1 + d1).
__device__ __forceinline__ void fma2_rn(float& d0, float& d1, float a0, float a1, float b0,
                                        float b1) {
  asm("{\n\t.reg .b64 pa, pb, pd;\n\t"
      "mov.b64 pa, {%2, %3};\n\t"
      "mov.b64 pb, {%4, %5};\n\t"
      "mov.b64 pd, {%0, %1};\n\t"
      "fma.rn.f32x2 pd, pa, pb, pd;\n\t"
      "mov.b64 {%0, %1}, pd;\n\t}"
      : "+f"(d0), "+f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

template <int D4, int RS, int LQ>
__device__ __forceinline__ void dots_fixed(const float* feat, const FeatLayout& Lf,
                                           const uint16_t* tiles, int S_here,
                                           float* __restrict__ out, int64_t b0,
                                           int64_t row_stride, int64_t col0, int tid,
                                           int nthreads) {
  constexpr int Q = 1 << LQ;
  constexpr int ITER = (D4 + Q - 1) / Q;
  const int total = (S_here * Lf.nT) << LQ;
  const int lane = tid & 31;
  const int per_sample = Lf.F1p * RS;
  for (int base = tid - lane; base < total; base += nthreads) {
    const int task = base + lane;
    const bool active = task < total;
    const int tt = active ? task : 0;
    const int q = tt & (Q - 1);
    const int rest = tt >> LQ;
    int t = rest, s = 0;
    if (S_here > 1) {
      s = rest / Lf.nT;
      t = rest - s * Lf.nT;
    }
    const int IJ = tiles[t];
    const int I = IJ >> 8, J = IJ & 255;
    const float4* fi = reinterpret_cast<const float4*>(feat) + s * per_sample + 4 * I * RS + q;
    const float4* fj = reinterpret_cast<const float4*>(feat) + s * per_sample + 4 * J * RS + q;
    float acc2[32];  // per dot, the partial sums of its even and of its odd columns
#pragma unroll
    for (int v = 0; v < 32; ++v) acc2[v] = 0.f;
#pragma unroll
    for (int it = 0; it < ITER; ++it) {
      if (it * Q + q < D4 || (D4 % Q) == 0) {
        float4 a[4], bv[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) a[r] = fi[r * RS + it * Q];
#pragma unroll
        for (int c = 0; c < 4; ++c) bv[c] = fj[c * RS + it * Q];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float& e = acc2[2 * (4 * r + c)];
            float& o = acc2[2 * (4 * r + c) + 1];
            fma2_rn(e, o, a[r].x, a[r].y, bv[c].x, bv[c].y);
            fma2_rn(e, o, a[r].z, a[r].w, bv[c].z, bv[c].w);
          }
      }
    }
    float acc[16];
#pragma unroll
    for (int v = 0; v < 16; ++v) acc[v] = acc2[2 * v] + acc2[2 * v + 1];
    tile_reduce_store<LQ>(acc, q, active, I, J, Lf.F1, out + (b0 + s) * row_stride + col0);
  }
}

// Bytes of the tile table decode_tiles writes (a multiple of 16).
__host__ __device__ inline int64_t tile_table_bytes(int nT) { return (2 * nT + 15) / 16 * 16; }

// The tile table sits in the last tile_table_bytes(nT) of the block's dynamic
// shared memory.
__device__ __forceinline__ uint16_t* tile_table(void* smem_base, int nT) {
  uint32_t total;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(total));
  return reinterpret_cast<uint16_t*>(static_cast<char*>(smem_base) + total -
                                     tile_table_bytes(nT));
}

// The dot phase of the interaction kernel: for the padded row length DP of
// the kernel instance (68 floats: D = 64; 132: D = 128) and four lanes per
// tile (the interaction launch's choice for those rows), the compile-time
// routine; dots_from_smem for the rest. Each instance holds only its own
// routine: with every fixed routine in every instance, instruction fetch was
// the kernel's largest stall. tiles is the table decode_tiles wrote (used by
// the fixed routine), or null when the block's shared memory has no room for
// it. (Measured on B200: in the interaction kernel the fixed routine took c3
// from 24.6 to 23.0 us; in the fused kernel, whose dot phase runs beside other
// blocks' gathers, it cost 2.5 us, so the fused kernel keeps dots_from_smem.)
template <int UNROLL, int DP>
__device__ __forceinline__ void dots_any(const float* feat, const FeatLayout& Lf,
                                         const uint16_t* tiles, int S_here, int lq,
                                         float* __restrict__ out, int64_t b0, int64_t row_stride,
                                         int64_t col0, int tid, int nthreads) {
  if constexpr (DP == 68) {
    if (tiles != nullptr && lq == 2 && Lf.D4 == 16 && Lf.Dp == 68) {
      dots_fixed<16, 17, 2>(feat, Lf, tiles, S_here, out, b0, row_stride, col0, tid, nthreads);
      return;
    }
  } else if constexpr (DP == 132) {
    if (tiles != nullptr && lq == 2 && Lf.D4 == 32 && Lf.Dp == 132) {
      dots_fixed<32, 33, 2>(feat, Lf, tiles, S_here, out, b0, row_stride, col0, tid, nthreads);
      return;
    }
  }
  dots_from_smem<UNROLL>(feat, Lf, S_here, lq, out, b0, row_stride, col0, tid, nthreads);
}

// Ampere-style asynchronous global -> shared copies (cp.async), used to stage
// the next group of samples while the current one is computed.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
// Wait until at most N of this thread's committed groups are still pending.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

}  // namespace dlrm
