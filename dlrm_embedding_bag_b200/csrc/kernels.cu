// The interaction-only kernel, the pair decoder, and the host-side choice of
// loader, template shape and block size for every launch (sm_100a).
//
//   embbag_kernel / fused_kernel : kernels.cuh, instantiated in inst_*.cu
//   interact_kernel    : strict-lower-triangle pairwise dots
//                        (dlrm_interact.rs, stacked kernel of the pages)
//   pair_decode_kernel : the closed-form pair decoders alone, for tests
#include <algorithm>
#include <atomic>

#include "interact_common.cuh"
#include "launch.h"
#include "tma_common.cuh"

namespace dlrm {

static std::atomic<int64_t> g_launches{0};

// Interaction alone. Persistent blocks walk groups of S samples (group g =
// blockIdx.x + i * gridDim.x); while the dots of one group run from one shared
// buffer, the [dense, emb] rows of the next group are copied into the other.
// Rows of whole 16-byte chunks (VEC = 4) arrive by bulk copies, one per feature
// row, counted on the buffer's mbarrier (stage_group_bulk); other rows by
// cp.async (below): warp w of W copies feature rows w, w + W, ...; when a row is
// at most 32 chunks of VEC floats and the chunk count divides 32, one warp copy
// covers 32/DV rows.
template <int VEC>
__device__ __forceinline__ void stage_interact_group(float* buf, const FeatLayout& Lf,
                                                     const float* __restrict__ dense,
                                                     const float* __restrict__ emb, int64_t b0,
                                                     int S_here, int F, int D) {
  const int DV = D / VEC;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  const bool packed = DV <= 32 && (32 % DV) == 0;
  const int rpw = packed ? 32 / DV : 1;              // rows per warp copy
  const int lr = packed ? lane / DV : 0;             // this lane's row within the copy
  const int c0 = packed ? (lane - lr * DV) : lane;  // this lane's first chunk
  const int cstep = packed ? DV : 32;
  for (int s = 0; s < S_here; ++s) {
    float* base = buf + s * Lf.floats_per_sample();
    const int64_t b = b0 + s;
    for (int f = warp * rpw + lr; f < Lf.F1; f += nwarps * rpw) {
      const float* src =
          (f == 0) ? dense + b * D : emb + (b * F + (f - 1)) * static_cast<int64_t>(D);
      float* dst = base + f * Lf.Dp;
      for (int c = c0; c < DV; c += cstep) {
        if constexpr (VEC == 4) {
          cp_async16(dst + 4 * c, src + 4 * c);
        } else {
          cp_async4(dst + c, src + c);
        }
      }
    }
  }
}

// The group's rows as one bulk copy each into the padded rows of `buf`
// (thread t copies rows t, t + nthreads, ...; D a multiple of 4 and both
// pointers 16-byte aligned); thread 0 announces the group's bytes on `bar`. The
// caller has synchronised the block after the buffer's last reads.
__device__ __forceinline__ void stage_group_bulk(float* buf, const FeatLayout& Lf,
                                                 const float* __restrict__ dense,
                                                 const float* __restrict__ emb, int64_t b0,
                                                 int S_here, int F, int D, uint64_t* bar) {
  const int rows = S_here * Lf.F1;
  const uint32_t row_bytes = static_cast<uint32_t>(D) * 4u;
  fence_proxy_async_smem();  // this thread's earlier reads of the buffer come first
  if (threadIdx.x == 0) mbar_arrive_expect_tx(bar, static_cast<uint32_t>(rows) * row_bytes);
  for (int t = threadIdx.x; t < rows; t += blockDim.x) {
    const int s = t / Lf.F1, f = t - s * Lf.F1;
    const int64_t b = b0 + s;
    const float* src =
        (f == 0) ? dense + b * D : emb + (b * F + (f - 1)) * static_cast<int64_t>(D);
    bulk_g2s(buf + s * Lf.floats_per_sample() + f * Lf.Dp, src, row_bytes, bar);
  }
}

// Blocks of the interaction kernel per SM (its register budget: 128 registers
// at 128-thread blocks; eight blocks would spill), and the unrolling of the
// general dot routine's column loop.
#ifndef DLRM_INTERACT_MIN_BLOCKS
#define DLRM_INTERACT_MIN_BLOCKS 4
#endif
#ifndef DLRM_INTERACT_UNROLL
#define DLRM_INTERACT_UNROLL 2
#endif

template <int VEC, int DP>
__global__ void __launch_bounds__(kBlockThreads, DLRM_INTERACT_MIN_BLOCKS)
    interact_kernel(const float* __restrict__ dense, const float* __restrict__ emb, int B, int F,
                    int D, int S, int lq, int nbuf, int with_tiles, float* __restrict__ out) {
  extern __shared__ __align__(16) float feat[];
  const FeatLayout Lf = FeatLayout::make(F, D);
  // buffer i at feat + i * bstride
  const int64_t bstride = (nbuf > 1) ? S * Lf.floats_per_sample() : 0;
  const int64_t ngroups = (static_cast<int64_t>(B) + S - 1) / S;
  const int P = Lf.F1 * (Lf.F1 - 1) / 2;
  auto samples = [&](int64_t g) {
    const int64_t rem = B - g * S;
    return rem < S ? static_cast<int>(rem) : S;
  };
  // The copies never write the padding, so it is zeroed once per buffer.
  for (int i = 0; i < nbuf; ++i)
    zero_feature_padding(feat + i * bstride, Lf, D, S, threadIdx.x, blockDim.x);
  uint16_t* tiles = with_tiles ? tile_table(feat, Lf.nT) : nullptr;
  if (tiles) decode_tiles(tiles, Lf.nT, threadIdx.x, blockDim.x);
  int64_t g = blockIdx.x;
  if (nbuf == 1) {
    for (; g < ngroups; g += gridDim.x) {
      stage_interact_group<VEC>(feat, Lf, dense, emb, g * S, samples(g), F, D);
      cp_async_commit();
      cp_async_wait<0>();
      __syncthreads();
      dots_any<DLRM_INTERACT_UNROLL, DP>(feat, Lf, tiles, samples(g), lq, out, g * S, P, 0,
                                     threadIdx.x, blockDim.x);
      __syncthreads();
    }
    return;
  }
  if constexpr (VEC == 4) {
    // two buffers with a barrier each: the i-th group of the block uses buffer
    // i & 1, whose (i >> 1)-th fill completes phase (i >> 1) of its barrier
    __shared__ __align__(8) uint64_t bars[2];
    if (threadIdx.x == 0) {
      mbar_init(&bars[0], 1);
      mbar_init(&bars[1], 1);
      mbar_init_fence();
    }
    __syncthreads();
    if (g < ngroups) stage_group_bulk(feat, Lf, dense, emb, g * S, samples(g), F, D, &bars[0]);
    for (int it = 0; g < ngroups; ++it, g += gridDim.x) {
      const int64_t gn = g + gridDim.x;
      if (gn < ngroups)
        stage_group_bulk(feat + ((it + 1) & 1) * bstride, Lf, dense, emb, gn * S, samples(gn), F,
                         D, &bars[(it + 1) & 1]);
      // bounded (about a second): the copies cannot stall, this only guards
      // the GPU against a broken barrier sequence
      mbar_wait_bounded(&bars[it & 1], (it >> 1) & 1, 2000000000LL);
      dots_any<DLRM_INTERACT_UNROLL, DP>(feat + (it & 1) * bstride, Lf, tiles, samples(g), lq, out,
                                     g * S, P, 0, threadIdx.x, blockDim.x);
      __syncthreads();  // buffer it & 1 is refilled in the next iteration
    }
    return;
  }
  if (g < ngroups) stage_interact_group<VEC>(feat, Lf, dense, emb, g * S, samples(g), F, D);
  cp_async_commit();
  for (int it = 0; g < ngroups; ++it, g += gridDim.x) {
    const int64_t gn = g + gridDim.x;
    if (gn < ngroups)
      stage_interact_group<VEC>(feat + ((it + 1) & 1) * bstride, Lf, dense, emb, gn * S,
                                samples(gn), F, D);
    cp_async_commit();
    cp_async_wait<1>();  // group g has landed (only the copy of group gn may be pending)
    __syncthreads();
    dots_any<DLRM_INTERACT_UNROLL, DP>(feat + (it & 1) * bstride, Lf, tiles, samples(g), lq, out,
                                   g * S, P, 0, threadIdx.x, blockDim.x);
    __syncthreads();  // buffer it&1 is refilled in the next iteration
  }
  cp_async_wait<0>();
}

// The bounded mbarrier wait of the asynchronous kernels, on a barrier that
// nothing completes (dlrm_probe_bounded_wait).
__global__ void probe_wait_kernel(long long limit, int32_t* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    mbar_init_fence();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait_bounded(&bar, 0, limit)) atomicOr(status, DLRM_FLAG_TIMEOUT);
}

// The random-row read probe (dlrm_probe_row_gather). Row n of the request
// stream is row splitmix64(seed + n) mod rows (Steele, Lea and Flood's
// SplitMix64 finaliser; the high half of a 64 x 64-bit product maps it onto
// [0, rows) without a division). A row of `chunks` 16-byte chunks is read by
// `chunks` consecutive lanes, 32 / chunks rows per warp at a time, eight such
// slots in flight before any value is used.
__device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
  x += 0x9E3779B97F4A7C15ull;
  x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
  x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
  return x ^ (x >> 31);
}

constexpr int kProbeThreads = 256;

__global__ void __launch_bounds__(kProbeThreads, 4)
    row_gather_probe_kernel(const uint4* __restrict__ table, int64_t rows, int lchunks,
                            int64_t count, uint64_t seed, uint32_t* __restrict__ sink) {
  constexpr int U = 8;
  const int chunks = 1 << lchunks;
  const int lane = threadIdx.x & 31;
  const int sub = lane >> lchunks, c = lane & (chunks - 1);
  const int per_warp = 32 >> lchunks;  // rows per warp slot
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t span = static_cast<int64_t>(per_warp) * U;
  uint32_t acc = 0;
  for (int64_t base = warp * span; base < count; base += nwarps * span) {
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t n = base + static_cast<int64_t>(u) * per_warp + sub;
      v[u] = make_uint4(0u, 0u, 0u, 0u);
      if (n < count) {
        const uint64_t row = __umul64hi(splitmix64(seed + static_cast<uint64_t>(n)),
                                        static_cast<uint64_t>(rows));
        const float4 f = ldg_row_f32x4(reinterpret_cast<const float*>(
            table + static_cast<int64_t>(row) * chunks + c));
        v[u] = make_uint4(__float_as_uint(f.x), __float_as_uint(f.y), __float_as_uint(f.z),
                          __float_as_uint(f.w));
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
  }
  if (acc == 0x2545F491u) atomicXor(sink, acc);
}

// Below 2^24 it runs pair_from_flat_small, the decoder dots_from_smem runs on
// the tile index in the interaction and fused kernels; from 2^24 on, the
// 64-bit pair_from_flat.
__global__ void pair_decode_kernel(int64_t p0, int64_t count, int32_t* __restrict__ i_out,
                                   int32_t* __restrict__ j_out) {
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < count;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t p = p0 + e;
    int i, j;
    if (p < kPairSmallLimit) {
      pair_from_flat_small(static_cast<int>(p), i, j);
    } else {
      pair_from_flat(p, i, j);
    }
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
    case kLdF32x4S: return 4;
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

// Samples per block of the fused kernel. A block's S*F bags go to its lane
// groups in rounds; measured on B200, blocks do best with at least two bags per
// lane group and little idle time in the last round, while blocks too large for
// DLRM_FUSED_MIN_BLOCKS of them to share an SM lose more than they gain (with
// 256-thread blocks, four per SM: B=65536, F=26, D=128 ran 12 % faster at S=2
// than at S=1). So: the smallest S up to 4 with >= 2 bags per group, >= 90 % of
// the rounds' slots used and DLRM_FUSED_MIN_BLOCKS blocks' shared memory
// fitting an SM; else the S with the best product of slot use and resident
// blocks. With 128-thread blocks: S = 1 at B=2048, F=32, D=64 and at B=65536,
// F=26, D=128; S = 2 at F=8, D=64.
#ifndef DLRM_FUSED_MAX_S
#define DLRM_FUSED_MAX_S 4
#endif
static int fused_samples_per_block(int F, int D, int B, int groups, int64_t extra_per_block) {
  const int64_t per = interact_smem_per_sample(F, D);
  const int64_t sm_bytes = 228 * 1024;
  int best_s = 1;
  double best = -1.0;
  for (int s = 1; s <= DLRM_FUSED_MAX_S && s <= B; ++s) {
    const int bags = s * F;
    const int rounds = (bags + groups - 1) / groups;
    const double util = static_cast<double>(bags) / (static_cast<double>(rounds) * groups);
    const int64_t resident = std::min<int64_t>(DLRM_FUSED_MIN_BLOCKS,
                                               sm_bytes / (s * per + extra_per_block + 1024));
    if (bags >= 2 * groups && util >= 0.9 && resident >= DLRM_FUSED_MIN_BLOCKS) return s;
    const double score = util * static_cast<double>(resident) / DLRM_FUSED_MIN_BLOCKS;
    if (score > best + 1e-9) {
      best = score;
      best_s = s;
    }
  }
  return best_s;
}

#ifndef DLRM_FUSED_LQ_MAX
#define DLRM_FUSED_LQ_MAX 4
#endif
// Samples per block and log2 of the lanes per tile for the dot phase.
static void choose_dot_shape(int F, int D, int B, int samples_wanted, int64_t smem_cap, int& S,
                             int& lq) {
  const FeatLayout Lf = FeatLayout::make(F, D);
  const int64_t per = Lf.floats_per_sample() * 4;
  int s = std::max(1, samples_wanted);
  s = static_cast<int>(std::min<int64_t>(s, std::max<int64_t>(1, smem_cap / per)));
  S = std::min(s, B);
  const int tiles = S * Lf.nT;
  // at least four lanes per tile, even when that takes the tasks more than one
  // round of the block's threads: with 128-thread blocks at B=2048, F=32, D=64
  // (45 tiles) two lanes per tile in one round ran 48.9 us and four lanes in two
  // rounds 46.5 us on B200 (bf16 tables 41.9 -> 39.9 us): a lane's 16 partial dots
  // are then fed by chunks of the same rows as three other lanes', which spreads
  // the shared-memory reads over the banks
  const int qmax = std::max(4, kBlockThreads / tiles);
  lq = std::min({log2_floor(qmax), log2_floor(std::max(1, Lf.D4)), DLRM_FUSED_LQ_MAX});
}

static cudaError_t counted(cudaError_t e) {
  if (e == cudaSuccess) g_launches.fetch_add(1, std::memory_order_relaxed);
  return e;
}

// --------------------------------------------------------------------------
// Path choice and the tensor-map encoder.

static std::atomic<int> g_path{DLRM_PATH_AUTO};
static thread_local int t_last_path = 0;
int gather_path() { return g_path.load(std::memory_order_relaxed); }
void set_gather_path(int path) { g_path.store(path, std::memory_order_relaxed); }
int last_path() { return t_last_path; }

// The driver's tensor-map encoder, looked up once through the runtime.
EncodeTiledFn encode_tiled() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

static int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n;
}


// One path serves every call: the per-block register-load kernels
// (DLRM_PATH_AUTO = DLRM_PATH_LDG).
cudaError_t launch_embbag(const GatherPlan& g, float* out, cudaStream_t stream) {
  const GatherShape sh = choose_gather_shape(g.D, g.loader);
  t_last_path = DLRM_PATH_LDG;
  GatherLaunch a{g.tp, g.bp, g.B, g.F, g.D, out, g.pool, sh, stream};
  switch (g.loader) {
    case kLdF32x4: return counted(launch_gather_f32x4(a));
    case kLdF32x4S: return counted(launch_gather_f32x4s(a));
    case kLdF32x1: return counted(launch_gather_f32x1(a));
    case kLdBF16x8: return counted(launch_gather_bf16x8(a));
    case kLdBF16x1: return counted(launch_gather_bf16x1(a));
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_fused(const GatherPlan& g, const float* dense, float* pooled_out,
                         float* inter_out, int concat_dense, int64_t smem_limit,
                         cudaStream_t stream) {
  t_last_path = DLRM_PATH_LDG;
  FusedLaunch a;
  a.g = GatherLaunch{g.tp, g.bp, g.B, g.F, g.D, nullptr, g.pool,
                     choose_gather_shape(g.D, g.loader), stream};
  a.dense = dense;
  a.pooled_out = pooled_out;
  a.inter_out = inter_out;
  a.concat_dense = concat_dense;
  const int groups = kBlockThreads / a.g.shape.G;
  // the bag ordering keeps 96 ints per warp after the features
  const int64_t order_bytes = a.g.bp.balance ? (kBlockThreads / 32) * 96 * sizeof(int) : 0;
  const int want = fused_samples_per_block(g.F, g.D, g.B, groups, order_bytes);
  choose_dot_shape(g.F, g.D, g.B, want, std::min<int64_t>(smem_limit, 64 * 1024) - order_bytes,
                   a.S, a.lq);
  if (a.S * g.F >= (1 << kSortTaskBits)) a.g.bp.balance = 0;
  // bag ordering only changes the order of work: drop it when its shared
  // memory would not fit next to the features
  if (a.g.bp.balance && a.S * interact_smem_per_sample(g.F, g.D) + order_bytes > smem_limit)
    a.g.bp.balance = 0;
  a.smem = a.S * interact_smem_per_sample(g.F, g.D) + (a.g.bp.balance ? order_bytes : 0);
  if (a.smem > smem_limit) return cudaErrorInvalidValue;
  switch (g.loader) {
    case kLdF32x4: return counted(launch_fused_f32x4(a));
    case kLdF32x4S: return counted(launch_fused_f32x4s(a));
    case kLdF32x1: return counted(launch_fused_f32x1(a));
    case kLdBF16x8: return counted(launch_fused_bf16x8(a));
    case kLdBF16x1: return counted(launch_fused_bf16x1(a));
    default: return cudaErrorInvalidValue;
  }
}

// Samples per group S and lanes per tile 2^lq for the interaction kernel.
// Measured on B200 (B=2048, F=32, D=64 and B=65536, F=26, D=128), four lanes
// per tile beat one or two (shorter serial chains per thread), and the best
// group is the largest that still gives one task per thread: S*nT*4 <= the
// block's threads (at least one sample).
// S is further capped by the shared-memory budget of two buffers.
static void choose_interact_shape(int F, int D, int B, int64_t smem_budget, int& S, int& lq) {
  const FeatLayout Lf = FeatLayout::make(F, D);
  const int64_t per = Lf.floats_per_sample() * 4;
  lq = std::min(2, log2_floor(std::max(1, Lf.D4)));
  S = std::max(1, kBlockThreads / std::max(1, Lf.nT << lq));
  while (S > 1 && 2 * S * per > smem_budget) --S;
  S = std::max(1, std::min(S, B));
}

template <int VEC, int DP>
static cudaError_t run_interact(const float* dense, const float* emb, int B, int F, int D,
                                float* out, int64_t smem_limit, int sms, cudaStream_t stream) {
  const FeatLayout Lf = FeatLayout::make(F, D);
  const int64_t per = Lf.floats_per_sample() * 4;
  if (per > smem_limit) return cudaErrorInvalidValue;
  auto* fn = &interact_kernel<VEC, DP>;
  const int64_t budget = std::min<int64_t>(smem_limit, 200 * 1024 / DLRM_INTERACT_MIN_BLOCKS);
  int S, lq;
  choose_interact_shape(F, D, B, budget, S, lq);
  // two buffers. Measured on B200 for the bulk-copy path (VEC = 4) against
  // cp.async, same call: B=65536, F=26, D=128 400 -> 337 us, B=2048, F=32, D=64
  // 19.4 -> 18.9 us; a ring of three or four buffers (more groups in flight)
  // measured slower (357 us and 20.7 us)
  const int nbuf = (2 * S * per <= smem_limit) ? 2 : 1;
  const int64_t tbytes = tile_table_bytes(Lf.nT);
  const int with_tiles = nbuf * S * per + tbytes <= smem_limit ? 1 : 0;
  const int64_t smem = nbuf * S * per + (with_tiles ? tbytes : 0);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(fn),
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  // threads: the group's tasks rounded up to whole warps, at most a full block
  // (with 256-thread blocks this took B=65536, F=26, D=128 from 447 to 398 us
  // on B200: 224 threads for 2 x 112 tasks)
  const int threads = std::min<int>(kBlockThreads, (S * (Lf.nT << lq) + 31) / 32 * 32);
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, threads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int64_t ngroups = (static_cast<int64_t>(B) + S - 1) / S;
  const int64_t grid = std::min<int64_t>(ngroups, static_cast<int64_t>(per_sm) * sms);
  fn<<<static_cast<unsigned>(grid), threads, smem, stream>>>(dense, emb, B, F, D, S, lq,
                                                                  nbuf, with_tiles, out);
  return cudaGetLastError();
}

cudaError_t launch_interact(const float* dense, const float* emb, int B, int F, int D, float* out,
                            bool vec_ok, int64_t smem_limit, cudaStream_t stream) {
  const int sms = sm_count();
  cudaError_t e;
  if (vec_ok && D == 64) {
    e = run_interact<4, 68>(dense, emb, B, F, D, out, smem_limit, sms, stream);
  } else if (vec_ok && D == 128) {
    e = run_interact<4, 132>(dense, emb, B, F, D, out, smem_limit, sms, stream);
  } else if (vec_ok) {
    e = run_interact<4, 0>(dense, emb, B, F, D, out, smem_limit, sms, stream);
  } else {
    e = run_interact<1, 0>(dense, emb, B, F, D, out, smem_limit, sms, stream);
  }
  return counted(e);
}

cudaError_t launch_probe_wait(int64_t limit, int32_t* status, cudaStream_t stream) {
  probe_wait_kernel<<<1, 32, 0, stream>>>(static_cast<long long>(limit), status);
  return counted(cudaGetLastError());
}

cudaError_t launch_probe_row_gather(const void* table, int64_t rows, int chunks, int64_t count,
                                    uint64_t seed, uint32_t* sink, cudaStream_t stream) {
  if (count == 0) return cudaSuccess;
  const int lchunks = log2_floor(chunks);
  row_gather_probe_kernel<<<static_cast<unsigned>(4 * sm_count()), kProbeThreads, 0, stream>>>(
      static_cast<const uint4*>(table), rows, lchunks, count, seed, sink);
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
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

}  // namespace dlrm
