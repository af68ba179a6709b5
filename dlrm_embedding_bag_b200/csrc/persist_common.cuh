// Shared pieces of the persistent gather kernels (sm_100a): the order in which
// a gather unit visits its bags, the feature-tile hand-over between gather
// warps and dot warps, and small store helpers.
#pragma once

#include "interact_common.cuh"
#include "tma_common.cuh"

namespace dlrm {

// Named barriers of the fused persistent kernels (0 is __syncthreads):
// READY p: gather warps arrive, dot warps wait -- feature tile p is complete;
// FREE p : dot warps arrive, gather warps wait -- feature tile p may be refilled.
enum { kBarReady0 = 1, kBarFree0 = 3 };

// Where a unit's bags come from.
//  fused  : the block's tiles lt = 0, 1, ... (tile t = blockIdx.x + lt*gridDim.x
//           of S samples); within a tile, bags j = u, u + units, ... of S_t*F.
//  gather : global bag ids g = blockIdx.x*units + u + i*gridDim.x*units.
struct BagPos {
  int valid, lt, j;  // j: bag within the tile (fused) or global bag id (gather)
  int b, k, start, n;
  bool bad;
};

template <bool FUSED>
struct BagOrder {
  int B, F, S, units, u, my_tiles;
  __device__ __forceinline__ int tile_samples(int lt) const {
    const int64_t t = static_cast<int64_t>(blockIdx.x) + static_cast<int64_t>(lt) * gridDim.x;
    const int64_t rem = B - t * S;
    return rem < S ? static_cast<int>(rem) : S;
  }
  __device__ __forceinline__ void first(BagPos& p) const {
    if (FUSED) {
      p.lt = 0;
      p.j = u;
      p.valid = 0;
      while (p.lt < my_tiles) {
        if (p.j < tile_samples(p.lt) * F) {
          p.valid = 1;
          break;
        }
        ++p.lt;
      }
    } else {
      p.lt = 0;
      p.j = static_cast<int>(blockIdx.x) * units + u;
      p.valid = static_cast<int64_t>(p.j) < static_cast<int64_t>(B) * F;
    }
  }
  __device__ __forceinline__ void next(const BagPos& c, BagPos& p) const {
    p = c;
    if (!c.valid) return;
    if (FUSED) {
      p.j = c.j + units;
      while (p.lt < my_tiles && p.j >= tile_samples(p.lt) * F) {
        ++p.lt;
        p.j = u;
      }
      p.valid = p.lt < my_tiles;
    } else {
      const int64_t g = static_cast<int64_t>(c.j) + static_cast<int64_t>(gridDim.x) * units;
      p.valid = g < static_cast<int64_t>(B) * F;
      p.j = p.valid ? static_cast<int>(g) : 0;
    }
  }
  // Fill b and k of a position.
  __device__ __forceinline__ void place(BagPos& p) const {
    if (!p.valid) {
      p.b = p.k = 0;
      return;
    }
    if (FUSED) {
      const int s = p.j / F;
      p.k = p.j - s * F;
      p.b = static_cast<int>((static_cast<int64_t>(blockIdx.x) +
                              static_cast<int64_t>(p.lt) * gridDim.x) * S) + s;
    } else {
      p.b = p.j / F;
      p.k = p.j - p.b * F;
    }
  }
  // Fill b, k and start the load of the bag's bounds.
  __device__ __forceinline__ void locate(BagPos& p, const BagParams& bp) const {
    place(p);
    if (!p.valid) {
      p.start = p.n = 0;
      p.bad = false;
      return;
    }
    bag_bounds(bp, B, p.k, p.b, p.start, p.n, p.bad);
  }
  // The raw offsets that bound a placed bag (loads only; see set_bounds).
  __device__ __forceinline__ void load_offsets(const BagPos& p, const BagParams& bp, int& s,
                                               int& e) const {
    if (!p.valid) {
      s = e = 0;
      return;
    }
    const int64_t o = static_cast<int64_t>(p.k) * (B + bp.ilo) + p.b;
    s = __ldg(bp.offsets + o);
    e = (bp.ilo || p.b + 1 < B) ? __ldg(bp.offsets + o + 1) : bp.T;
  }
  // Bounds from raw offsets, with the same validity rule as bag_bounds.
  __device__ __forceinline__ static void set_bounds(BagPos& p, int s, int e, int T) {
    p.bad = p.valid && ((s < 0) || (s > e) || (e > T));
    p.start = p.bad ? 0 : s;
    p.n = (p.bad || !p.valid) ? 0 : e - s;
  }
};

template <int VEC>
__device__ __forceinline__ void store_vec_f32(float* p, const float (&a)[VEC]) {
#pragma unroll
  for (int e = 0; e < VEC; e += 4)
    *reinterpret_cast<float4*>(p + e) = make_float4(a[e], a[e + 1], a[e + 2], a[e + 3]);
}

// The dot warps of a fused persistent kernel: for each of the block's tiles,
// stage the dense rows into feature tile lt&1, wait until the gather warps
// have pooled the tile, copy the dense part of concatenated rows, compute the
// dots, and hand the tile back. Threads [NGW*32, (NGW+NDW)*32) of the block.
template <int NGW, int NDW>
__device__ __forceinline__ void fused_dot_warps(float* feat, const FeatLayout& Lf,
                                                const float* __restrict__ dense, int B, int D,
                                                int S, int lq, int my_tiles,
                                                float* __restrict__ inter_out,
                                                int concat_dense) {
  constexpr int NT = (NGW + NDW) * 32;
  constexpr int nthr = NDW * 32;
  const int tid = threadIdx.x - NGW * 32;
  const int64_t sample_floats = Lf.floats_per_sample();
  const int64_t P = static_cast<int64_t>(Lf.F1) * (Lf.F1 - 1) / 2;
  const int64_t row_stride = concat_dense ? D + P : P;
  const bool dense_vec = ((D & 3) == 0) && ((reinterpret_cast<uintptr_t>(dense) & 15) == 0);
  for (int lt = 0; lt < my_tiles; ++lt) {
    const int p = lt & 1;
    float* fb = feat + p * S * sample_floats;
    const int64_t b0 =
        (static_cast<int64_t>(blockIdx.x) + static_cast<int64_t>(lt) * gridDim.x) * S;
    const int S_t = (B - b0 < S) ? static_cast<int>(B - b0) : S;
    for (int s = 0; s < S_t; ++s) {
      const float* src = dense + (b0 + s) * D;
      float* dst = fb + s * sample_floats;
      if (dense_vec) {
        for (int c4 = tid; c4 < (D >> 2); c4 += nthr)
          reinterpret_cast<float4*>(dst)[c4] = __ldg(reinterpret_cast<const float4*>(src) + c4);
      } else {
        for (int c1 = tid; c1 < D; c1 += nthr) dst[c1] = __ldg(src + c1);
      }
    }
    zero_feature_padding(fb, Lf, D, S_t, tid, nthr);
    named_bar_sync(kBarReady0 + p, NT);
    if (concat_dense) {
      for (int s = 0; s < S_t; ++s) {
        const float* src = fb + s * sample_floats;
        float* dst = inter_out + (b0 + s) * row_stride;
        for (int d = tid; d < D; d += nthr) dst[d] = src[d];
      }
    }
    dots_from_smem(fb, Lf, S_t, lq, inter_out, b0, row_stride, concat_dense ? D : 0, tid, nthr);
    if (lt + 2 < my_tiles) named_bar_arrive(kBarFree0 + p, NT);
  }
}

// Tiles of S samples owned by this block (tile t = blockIdx.x + lt*gridDim.x).
__device__ __forceinline__ int block_tiles(int B, int S) {
  const int64_t ntiles = (static_cast<int64_t>(B) + S - 1) / S;
  return blockIdx.x < ntiles ? static_cast<int>((ntiles - 1 - blockIdx.x) / gridDim.x + 1) : 0;
}

}  // namespace dlrm
