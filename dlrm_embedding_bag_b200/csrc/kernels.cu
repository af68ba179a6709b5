// Kernels of the DLRMv1 sparse/interaction stage for B200 (sm_100a), and the
// launchers that pick their template shape.
//
//   embbag_kernel   : multi-table EmbeddingBag sum, one launch for all tables
//                     (embedding_bag.rs, multi-table section of the pages).
//   interact_kernel : strict-lower-triangle pairwise dots
//                     (dlrm_interact.rs, stacked kernel of the pages).
//   fused_kernel    : both, with the pooled vectors kept in shared memory.
//   pair_decode_kernel : the closed-form pair decoder alone, for tests.
#include <algorithm>
#include <atomic>

#include "interact_common.cuh"
#include "launch.h"

namespace dlrm {

std::atomic<int64_t> g_launches{0};

// --------------------------------------------------------------------------
// Gather: one lane group of G lanes per bag (b, k); bag id u = b*F + k, so
// consecutive groups write consecutive pooled vectors.
template <int VEC, int G, int CPL, int U, bool CHECK>
__global__ void __launch_bounds__(kBlockThreads)
    embbag_kernel(const __grid_constant__ TableParams tp, const int32_t* __restrict__ indices,
                  const int32_t* __restrict__ offsets, int B, int F, int L, int D, int ncolwin,
                  float* __restrict__ out, int32_t* __restrict__ status) {
  using V = typename VecOf<VEC>::T;
  constexpr int kGroups = kBlockThreads / G;
  const int lane = threadIdx.x & 31;
  const int q = lane % G;
  const int gbase = lane - q;
  const int BL = B * L;
  const int64_t bag = static_cast<int64_t>(blockIdx.x) * kGroups + threadIdx.x / G;
  const bool active = bag < static_cast<int64_t>(B) * F;
  if (__all_sync(kFullMask, !active)) return;

  const int b = active ? static_cast<int>(bag / F) : 0;
  const int k = active ? static_cast<int>(bag - static_cast<int64_t>(b) * F) : 0;
  int start = 0, n = 0;
  bool bad = false;
  if (active) bag_bounds(offsets, B, BL, k, b, start, n, bad);
  const int nmax = __reduce_max_sync(kFullMask, n);
  const float* W = tp.w[k];
  const int32_t* idx_seg = indices + static_cast<int64_t>(k) * BL;
  const int rows_k = CHECK ? tp.rows[k] : 0;
  bool oob = false;
  float* orow = out + (static_cast<int64_t>(b) * F + k) * D;

  for (int w = 0; w < ncolwin; ++w) {
    const int col0 = w * (G * CPL * VEC);
    V acc[CPL];
    pool_bag<VEC, G, CPL, U, CHECK>(W, rows_k, idx_seg, start, n, nmax, D, col0, q, gbase, acc,
                                    oob);
    if (active) {
#pragma unroll
      for (int m = 0; m < CPL; ++m) {
        const int col = col0 + (q + G * m) * VEC;
        if (col < D) store_vec(orow + col, acc[m]);
      }
    }
  }
  if (CHECK && status != nullptr) {
    const int flags = (oob ? DLRM_FLAG_INDEX_OOB : 0) | (bad ? DLRM_FLAG_OFFSETS : 0);
    if (flags) atomicOr(status, flags);
  }
}

// --------------------------------------------------------------------------
// Interaction alone: each block stages S samples' [dense, emb] rows in shared
// memory with coalesced loads, then runs the tiled dot phase.
template <int VEC>
__global__ void __launch_bounds__(kBlockThreads)
    interact_kernel(const float* __restrict__ dense, const float* __restrict__ emb, int B, int F,
                    int D, int S, int Q, float* __restrict__ out) {
  using V = typename VecOf<VEC>::T;
  extern __shared__ __align__(16) float feat[];
  const FeatLayout Lf = FeatLayout::make(F, D);
  const int64_t b0 = static_cast<int64_t>(blockIdx.x) * S;
  const int S_here = (B - b0 < S) ? static_cast<int>(B - b0) : S;
  const int DV = D / VEC;
  const int per_sample = Lf.F1 * DV;
  for (int e = threadIdx.x; e < S_here * per_sample; e += blockDim.x) {
    const int s = e / per_sample;
    const int rem = e - s * per_sample;
    const int f = rem / DV;
    const int c = (rem - f * DV) * VEC;
    const float* src = (f == 0) ? dense + (b0 + s) * D + c
                                : emb + ((b0 + s) * F + (f - 1)) * static_cast<int64_t>(D) + c;
    store_vec(feat + (static_cast<int64_t>(s) * Lf.F1p + f) * Lf.Dp + c,
              load_row_chunk(src, static_cast<V*>(nullptr)));
  }
  zero_feature_padding(feat, Lf, D, S_here);
  __syncthreads();
  const int P = Lf.F1 * (Lf.F1 - 1) / 2;
  dots_from_smem(feat, Lf, S_here, Q, out, b0, P, 0);
}

// --------------------------------------------------------------------------
// Fused: each block owns S consecutive samples. Phase 1 gathers their S*F
// bags straight into shared memory (and, if asked, to pooled_out) next to the
// dense rows; phase 2 computes the dots from shared memory. Only pooled_out
// and inter_out are written to global memory.
template <int VEC, int G, int CPL, int U, bool CHECK>
__global__ void __launch_bounds__(kBlockThreads)
    fused_kernel(const __grid_constant__ TableParams tp, const int32_t* __restrict__ indices,
                 const int32_t* __restrict__ offsets, const float* __restrict__ dense, int B,
                 int F, int L, int D, int ncolwin, int S, int Q, float* __restrict__ pooled_out,
                 float* __restrict__ inter_out, int concat_dense, int32_t* __restrict__ status) {
  using V = typename VecOf<VEC>::T;
  extern __shared__ __align__(16) float feat[];
  constexpr int kGroups = kBlockThreads / G;
  const FeatLayout Lf = FeatLayout::make(F, D);
  const int64_t b0 = static_cast<int64_t>(blockIdx.x) * S;
  const int S_here = (B - b0 < S) ? static_cast<int>(B - b0) : S;
  const int BL = B * L;
  const int lane = threadIdx.x & 31;
  const int q = lane % G;
  const int gbase = lane - q;

  // dense rows -> feature row 0
  const int DV = D / VEC;
  for (int e = threadIdx.x; e < S_here * DV; e += blockDim.x) {
    const int s = e / DV;
    const int c = (e - s * DV) * VEC;
    store_vec(feat + static_cast<int64_t>(s) * Lf.F1p * Lf.Dp + c,
              load_row_chunk(dense + (b0 + s) * D + c, static_cast<V*>(nullptr)));
  }
  zero_feature_padding(feat, Lf, D, S_here);

  // bags (s, k) -> feature row k + 1; every group runs the same number of rounds
  bool oob = false, bad_any = false;
  const int ntasks = S_here * F;
  const int rounds = (S * F + kGroups - 1) / kGroups;
  for (int rd = 0; rd < rounds; ++rd) {
    const int task = rd * kGroups + static_cast<int>(threadIdx.x) / G;
    const bool active = task < ntasks;
    const int s = active ? task / F : 0;
    const int k = active ? task - s * F : 0;
    int start = 0, n = 0;
    bool bad = false;
    if (active) bag_bounds(offsets, B, BL, k, static_cast<int>(b0 + s), start, n, bad);
    bad_any |= bad;
    const int nmax = __reduce_max_sync(kFullMask, n);
    const float* W = tp.w[k];
    const int32_t* idx_seg = indices + static_cast<int64_t>(k) * BL;
    const int rows_k = CHECK ? tp.rows[k] : 0;
    float* frow = feat + (static_cast<int64_t>(s) * Lf.F1p + 1 + k) * Lf.Dp;
    float* prow = pooled_out ? pooled_out + ((b0 + s) * F + k) * static_cast<int64_t>(D)
                             : nullptr;
    for (int w = 0; w < ncolwin; ++w) {
      const int col0 = w * (G * CPL * VEC);
      V acc[CPL];
      pool_bag<VEC, G, CPL, U, CHECK>(W, rows_k, idx_seg, start, n, nmax, D, col0, q, gbase,
                                      acc, oob);
      if (active) {
#pragma unroll
        for (int m = 0; m < CPL; ++m) {
          const int col = col0 + (q + G * m) * VEC;
          if (col < D) {
            store_vec(frow + col, acc[m]);
            if (prow) store_vec(prow + col, acc[m]);
          }
        }
      }
    }
  }
  if (CHECK && status != nullptr) {
    const int flags = (oob ? DLRM_FLAG_INDEX_OOB : 0) | (bad_any ? DLRM_FLAG_OFFSETS : 0);
    if (flags) atomicOr(status, flags);
  }
  __syncthreads();

  const int64_t P = static_cast<int64_t>(Lf.F1) * (Lf.F1 - 1) / 2;
  const int64_t row_stride = concat_dense ? D + P : P;
  if (concat_dense) {
    for (int e = threadIdx.x; e < S_here * D; e += blockDim.x) {
      const int s = e / D;
      const int d = e - s * D;
      inter_out[(b0 + s) * row_stride + d] = feat[static_cast<int64_t>(s) * Lf.F1p * Lf.Dp + d];
    }
  }
  dots_from_smem(feat, Lf, S_here, Q, inter_out, b0, row_stride, concat_dense ? D : 0);
}

// --------------------------------------------------------------------------
__global__ void pair_decode_kernel(int64_t p0, int64_t count, int32_t* __restrict__ i_out,
                                   int32_t* __restrict__ j_out) {
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < count;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    int i, j;
    pair_from_flat(p0 + e, i, j);
    i_out[e] = i;
    j_out[e] = j;
  }
}

// ==========================================================================
// Host side: shape selection and template dispatch.

static int pow2_ceil(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}
static int pow2_floor(int x) {
  int p = 1;
  while (p * 2 <= x) p <<= 1;
  return p;
}

GatherShape choose_gather_shape(int D, bool vec_ok) {
  GatherShape g;
  g.vec = vec_ok ? 4 : 1;
  const int chunks = D / g.vec;  // exact for vec 4 (D % 4 == 0)
  g.G = std::min(32, pow2_ceil(chunks));
  g.cpl = chunks > 32 ? 2 : 1;
  g.u = g.cpl == 1 ? 16 : 8;
  const int window = g.G * g.cpl * g.vec;
  g.ncolwin = (D + window - 1) / window;
  return g;
}

int64_t interact_smem_per_sample(int F, int D) {
  return FeatLayout::make(F, D).floats_per_sample() * static_cast<int64_t>(sizeof(float));
}

// Calls f.template run<VEC, G, CPL, U, CHECK>() for the runtime shape.
template <typename Fn>
static cudaError_t dispatch_gather(const GatherShape& g, bool check, Fn&& f) {
#define DLRM_CASE(V_, G_, C_, U_)                                         \
  if (g.vec == V_ && g.G == G_ && g.cpl == C_ && g.u == U_) {             \
    return check ? f.template run<V_, G_, C_, U_, true>()                 \
                 : f.template run<V_, G_, C_, U_, false>();               \
  }
  DLRM_CASE(4, 1, 1, 16)
  DLRM_CASE(4, 2, 1, 16)
  DLRM_CASE(4, 4, 1, 16)
  DLRM_CASE(4, 8, 1, 16)
  DLRM_CASE(4, 16, 1, 16)
  DLRM_CASE(4, 32, 1, 16)
  DLRM_CASE(4, 32, 2, 8)
  DLRM_CASE(1, 1, 1, 16)
  DLRM_CASE(1, 2, 1, 16)
  DLRM_CASE(1, 4, 1, 16)
  DLRM_CASE(1, 8, 1, 16)
  DLRM_CASE(1, 16, 1, 16)
  DLRM_CASE(1, 32, 1, 16)
  DLRM_CASE(1, 32, 2, 8)
#undef DLRM_CASE
  return cudaErrorInvalidConfiguration;
}

static cudaError_t finish_launch() {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError();
}

struct EmbbagRun {
  const TableParams& tp;
  const int32_t* indices;
  const int32_t* offsets;
  int B, F, L, D, ncolwin;
  float* out;
  int32_t* status;
  int64_t grid;
  cudaStream_t stream;
  template <int VEC, int G, int CPL, int U, bool CHECK>
  cudaError_t run() {
    embbag_kernel<VEC, G, CPL, U, CHECK><<<static_cast<unsigned>(grid), kBlockThreads, 0,
                                           stream>>>(tp, indices, offsets, B, F, L, D, ncolwin,
                                                     out, status);
    return finish_launch();
  }
};

cudaError_t launch_embbag(const TableParams& tp, const int32_t* indices, const int32_t* offsets,
                          int B, int F, int L, int D, float* out, int32_t* status, bool check,
                          bool vec_ok, cudaStream_t stream) {
  const GatherShape g = choose_gather_shape(D, vec_ok);
  const int groups = kBlockThreads / g.G;
  const int64_t nbags = static_cast<int64_t>(B) * F;
  const int64_t grid = (nbags + groups - 1) / groups;
  if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
  EmbbagRun r{tp, indices, offsets, B, F, L, D, g.ncolwin, out, status, grid, stream};
  return dispatch_gather(g, check, r);
}

// Samples per block and lanes per tile for the dot phase.
static void choose_dot_shape(int F, int D, int B, int samples_wanted, int64_t smem_limit, int& S,
                             int& Q) {
  const FeatLayout Lf = FeatLayout::make(F, D);
  const int64_t per = Lf.floats_per_sample() * 4;
  int s = std::max(1, samples_wanted);
  s = static_cast<int>(std::min<int64_t>(s, std::max<int64_t>(1, smem_limit / per)));
  s = std::min(s, B);
  S = s;
  const int tiles = S * Lf.nT;
  int qmax = std::max(1, kBlockThreads / tiles);
  Q = std::min({pow2_floor(qmax), pow2_floor(std::max(1, Lf.D4)), 32});
}

static cudaError_t set_smem(const void* fn, int64_t bytes) {
  if (bytes > 48 * 1024) {
    return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(bytes));
  }
  return cudaSuccess;
}

cudaError_t launch_interact(const float* dense, const float* emb, int B, int F, int D, float* out,
                            bool vec_ok, int64_t smem_limit, cudaStream_t stream) {
  int S, Q;
  // enough samples that the staging loop and the dot phase keep 256 threads busy
  const FeatLayout Lf = FeatLayout::make(F, D);
  const int want = std::max(1, kBlockThreads / std::max(1, Lf.nT * std::min(Lf.D4, 4)));
  choose_dot_shape(F, D, B, std::min(want, 8), std::min<int64_t>(smem_limit, 64 * 1024), S, Q);
  const int64_t smem = S * Lf.floats_per_sample() * 4;
  if (smem > smem_limit) return cudaErrorInvalidValue;
  const int64_t grid = (static_cast<int64_t>(B) + S - 1) / S;
  cudaError_t e;
  if (vec_ok) {
    if ((e = set_smem(reinterpret_cast<const void*>(&interact_kernel<4>), smem)) != cudaSuccess)
      return e;
    interact_kernel<4><<<static_cast<unsigned>(grid), kBlockThreads, smem, stream>>>(
        dense, emb, B, F, D, S, Q, out);
  } else {
    if ((e = set_smem(reinterpret_cast<const void*>(&interact_kernel<1>), smem)) != cudaSuccess)
      return e;
    interact_kernel<1><<<static_cast<unsigned>(grid), kBlockThreads, smem, stream>>>(
        dense, emb, B, F, D, S, Q, out);
  }
  return finish_launch();
}

struct FusedRun {
  const TableParams& tp;
  const int32_t* indices;
  const int32_t* offsets;
  const float* dense;
  int B, F, L, D, ncolwin, S, Q;
  float* pooled_out;
  float* inter_out;
  int concat_dense;
  int32_t* status;
  int64_t grid, smem;
  cudaStream_t stream;
  template <int VEC, int G, int CPL, int U, bool CHECK>
  cudaError_t run() {
    auto* fn = &fused_kernel<VEC, G, CPL, U, CHECK>;
    cudaError_t e = set_smem(reinterpret_cast<const void*>(fn), smem);
    if (e != cudaSuccess) return e;
    fn<<<static_cast<unsigned>(grid), kBlockThreads, smem, stream>>>(
        tp, indices, offsets, dense, B, F, L, D, ncolwin, S, Q, pooled_out, inter_out,
        concat_dense, status);
    return finish_launch();
  }
};

cudaError_t launch_fused(const TableParams& tp, const int32_t* indices, const int32_t* offsets,
                         const float* dense, int B, int F, int L, int D, float* pooled_out,
                         float* inter_out, int concat_dense, int32_t* status, bool check,
                         bool vec_ok, int64_t smem_limit, cudaStream_t stream) {
  const GatherShape g = choose_gather_shape(D, vec_ok);
  const int groups = kBlockThreads / g.G;
  // enough samples that every lane group has a bag in the gather phase
  const int want = std::max(1, (groups + F - 1) / F);
  int S, Q;
  choose_dot_shape(F, D, B, std::min(want, 16), std::min<int64_t>(smem_limit, 64 * 1024), S, Q);
  const FeatLayout Lf = FeatLayout::make(F, D);
  const int64_t smem = S * Lf.floats_per_sample() * 4;
  if (smem > smem_limit) return cudaErrorInvalidValue;
  const int64_t grid = (static_cast<int64_t>(B) + S - 1) / S;
  FusedRun r{tp, indices, offsets, dense, B, F, L, D, g.ncolwin, S, Q, pooled_out, inter_out,
             concat_dense, status, grid, smem, stream};
  return dispatch_gather(g, check, r);
}

cudaError_t launch_pair_decode(int64_t p0, int64_t count, int32_t* i_out, int32_t* j_out,
                               cudaStream_t stream) {
  if (count == 0) return cudaSuccess;
  const int64_t blocks = std::min<int64_t>((count + kBlockThreads - 1) / kBlockThreads, 148 * 16);
  pair_decode_kernel<<<static_cast<unsigned>(blocks), kBlockThreads, 0, stream>>>(p0, count,
                                                                                 i_out, j_out);
  return finish_launch();
}

int64_t launch_count() { return g_launches.load(std::memory_order_relaxed); }

}  // namespace dlrm
