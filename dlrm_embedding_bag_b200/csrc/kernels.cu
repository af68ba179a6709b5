// The interaction-only kernel, the pair decoder, and the host-side choice of
// loader, template shape and block size for every launch (sm_100a).
//
//   embbag_kernel / fused_kernel : kernels.cuh, instantiated in inst_*.cu
//   interact_kernel    : strict-lower-triangle pairwise dots
//                        (dlrm_interact.rs, stacked kernel of the pages)
//   pair_decode_kernel : the closed-form pair decoder alone, for tests
#include <algorithm>
#include <atomic>

#include "interact_common.cuh"
#include "launch.h"

namespace dlrm {

static std::atomic<int64_t> g_launches{0};

// Interaction alone: each block stages S samples' [dense, emb] rows in shared
// memory with coalesced loads, then runs the tiled dot phase.
template <int VEC>
__global__ void __launch_bounds__(kBlockThreads)
    interact_kernel(const float* __restrict__ dense, const float* __restrict__ emb, int B, int F,
                    int D, int S, int lq, float* __restrict__ out) {
  extern __shared__ __align__(16) float feat[];
  const FeatLayout Lf = FeatLayout::make(F, D);
  const int64_t b0 = static_cast<int64_t>(blockIdx.x) * S;
  const int S_here = (B - b0 < S) ? static_cast<int>(B - b0) : S;
  const int DV = D / VEC;
  const int per_sample = Lf.F1 * DV;
  for (int s = 0; s < S_here; ++s) {
    float* base = feat + s * Lf.floats_per_sample();
    for (int e = threadIdx.x; e < per_sample; e += blockDim.x) {
      const int f = e / DV;
      const int c = (e - f * DV) * VEC;
      const float* src = (f == 0) ? dense + (b0 + s) * D + c
                                  : emb + ((b0 + s) * F + (f - 1)) * static_cast<int64_t>(D) + c;
      if constexpr (VEC == 4) {
        *reinterpret_cast<float4*>(base + f * Lf.Dp + c) =
            __ldg(reinterpret_cast<const float4*>(src));
      } else {
        base[f * Lf.Dp + c] = __ldg(src);
      }
    }
  }
  zero_feature_padding(feat, Lf, D, S_here);
  __syncthreads();
  const int P = Lf.F1 * (Lf.F1 - 1) / 2;
  dots_from_smem(feat, Lf, S_here, lq, out, b0, P, 0);
}

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
// Host side.

static int pow2_ceil(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}
static int log2_floor(int x) {
  int l = 0;
  while ((2 << l) <= x) ++l;
  return l;
}

static int loader_vec(int loader) {
  switch (loader) {
    case kLdF32x4: return 4;
    case kLdBF16x8: return 8;
    default: return 1;
  }
}

GatherShape choose_gather_shape(int D, int loader) {
  GatherShape g;
  g.loader = loader;
  g.vec = loader_vec(loader);
  const int chunks = (D + g.vec - 1) / g.vec;  // exact for the vector loaders
  g.G = std::min(32, std::max(4, pow2_ceil(chunks)));
  g.cpl = chunks > 32 ? 2 : 1;
  const int window = g.G * g.cpl * g.vec;
  g.ncolwin = (D + window - 1) / window;
  return g;
}

int64_t interact_smem_per_sample(int F, int D) {
  return FeatLayout::make(F, D).floats_per_sample() * static_cast<int64_t>(sizeof(float));
}

// Samples per block and log2 of the lanes per tile for the dot phase.
static void choose_dot_shape(int F, int D, int B, int samples_wanted, int64_t smem_cap, int& S,
                             int& lq) {
  const FeatLayout Lf = FeatLayout::make(F, D);
  const int64_t per = Lf.floats_per_sample() * 4;
  int s = std::max(1, samples_wanted);
  s = static_cast<int>(std::min<int64_t>(s, std::max<int64_t>(1, smem_cap / per)));
  S = std::min(s, B);
  const int tiles = S * Lf.nT;
  const int qmax = std::max(1, kBlockThreads / tiles);
  lq = std::min({log2_floor(qmax), log2_floor(std::max(1, Lf.D4)), 5});
}

static cudaError_t counted(cudaError_t e) {
  if (e == cudaSuccess) g_launches.fetch_add(1, std::memory_order_relaxed);
  return e;
}

cudaError_t launch_embbag(const TableParams& tp, const BagParams& bp, int B, int F, int D,
                          float* out, int pool, int loader, cudaStream_t stream) {
  GatherLaunch a{&tp, bp, B, F, D, out, pool, choose_gather_shape(D, loader), stream};
  switch (loader) {
    case kLdF32x4: return counted(launch_gather_f32x4(a));
    case kLdF32x1: return counted(launch_gather_f32x1(a));
    case kLdBF16x8: return counted(launch_gather_bf16x8(a));
    case kLdBF16x1: return counted(launch_gather_bf16x1(a));
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_fused(const TableParams& tp, const BagParams& bp, const float* dense, int B,
                         int F, int D, float* pooled_out, float* inter_out, int concat_dense,
                         int pool, int loader, int64_t smem_limit, cudaStream_t stream) {
  FusedLaunch a;
  a.g = GatherLaunch{&tp, bp, B, F, D, nullptr, pool, choose_gather_shape(D, loader), stream};
  a.dense = dense;
  a.pooled_out = pooled_out;
  a.inter_out = inter_out;
  a.concat_dense = concat_dense;
  // enough samples that every lane group has a bag in the gather phase
  const int groups = kBlockThreads / a.g.shape.G;
  const int want = std::max(1, (groups + F - 1) / F);
  choose_dot_shape(F, D, B, std::min(want, 16), std::min<int64_t>(smem_limit, 64 * 1024), a.S,
                   a.lq);
  a.smem = a.S * interact_smem_per_sample(F, D);
  if (a.smem > smem_limit) return cudaErrorInvalidValue;
  switch (loader) {
    case kLdF32x4: return counted(launch_fused_f32x4(a));
    case kLdF32x1: return counted(launch_fused_f32x1(a));
    case kLdBF16x8: return counted(launch_fused_bf16x8(a));
    case kLdBF16x1: return counted(launch_fused_bf16x1(a));
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_interact(const float* dense, const float* emb, int B, int F, int D, float* out,
                            bool vec_ok, int64_t smem_limit, cudaStream_t stream) {
  const FeatLayout Lf = FeatLayout::make(F, D);
  // enough samples that the staging loop and the dot phase keep 256 threads busy
  const int want = std::max(1, kBlockThreads / std::max(1, Lf.nT * std::min(Lf.D4, 4)));
  int S, lq;
  choose_dot_shape(F, D, B, std::min(want, 8), std::min<int64_t>(smem_limit, 64 * 1024), S, lq);
  const int64_t smem = S * Lf.floats_per_sample() * 4;
  if (smem > smem_limit) return cudaErrorInvalidValue;
  const int64_t grid = (static_cast<int64_t>(B) + S - 1) / S;
  const void* fn = vec_ok ? reinterpret_cast<const void*>(&interact_kernel<4>)
                          : reinterpret_cast<const void*>(&interact_kernel<1>);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  if (vec_ok) {
    interact_kernel<4><<<static_cast<unsigned>(grid), kBlockThreads, smem, stream>>>(
        dense, emb, B, F, D, S, lq, out);
  } else {
    interact_kernel<1><<<static_cast<unsigned>(grid), kBlockThreads, smem, stream>>>(
        dense, emb, B, F, D, S, lq, out);
  }
  return counted(cudaGetLastError());
}

cudaError_t launch_pair_decode(int64_t p0, int64_t count, int32_t* i_out, int32_t* j_out,
                               cudaStream_t stream) {
  if (count == 0) return cudaSuccess;
  const int64_t blocks = std::min<int64_t>((count + kBlockThreads - 1) / kBlockThreads, 148 * 16);
  pair_decode_kernel<<<static_cast<unsigned>(blocks), kBlockThreads, 0, stream>>>(p0, count,
                                                                                 i_out, j_out);
  return counted(cudaGetLastError());
}

int64_t launch_count() { return g_launches.load(std::memory_order_relaxed); }

}  // namespace dlrm
