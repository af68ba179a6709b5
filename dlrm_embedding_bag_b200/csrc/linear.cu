// DLRMv1 MLP layer on the sm_100a tensor cores: Y = act([A_lo | A_hi] W^T + bias)
// (luminal compare main...vanilla-pytorch, matmul2d.rs: linear_bias,
// linear_bias_relu, linear_bias_sigmoid and the split-A forms), plus the f32 ->
// bf16 conversion that feeds it. Declared in dlrm_mlp.h.
//
// Persistent, warp-specialised kernel: CTA c walks the 128 x BN tiles
// t = c, c + gridDim.x, ... (N tiles fastest, so CTAs running side by side
// share A rows in L2). Ten warps:
//   - warp 0 (one thread) streams 64-wide K blocks of A (128 x 64 bf16) and W
//     (BN x 64) into a shared-memory ring (3 to 6 stages, by stage size) with 2-D
//     TMA loads (128-byte swizzle), running ahead across tiles; K blocks
//     0..nkb_lo-1 read A_lo, the rest read A_hi, and W's column offset follows,
//     so the concatenation is never built. An f32-activation operand is three
//     bf16 planes: a stage holds a K block's three plane boxes next to the W
//     box they share;
//   - warp 1 allocates tensor memory for two f32 accumulators (2 x BN
//     columns) and one thread issues four tcgen05.mma (K = 16 each) per A box
//     of a stage into the tile's accumulator, committing each stage back to
//     the producer and each finished accumulator to the epilogue;
//   - warps 2-9 read the finished accumulator (warp w owns TMEM lanes
//     32*(w%4)..+31 and half of the columns), add the bias, apply the
//     activation and store f32 and/or bf16, then hand the accumulator back -
//     so the epilogue of tile i runs while the MMAs of tile i+1 fill the
//     other accumulator.
// Large layers run the same roles on CTA pairs (clusters of two, tcgen05
// cta_group::2): a pair owns 256 x BN tiles, each CTA loads its 128 rows of A
// and half of the tile's W rows per stage, the even CTA issues M = 256 MMAs
// over both CTAs' shared memory, and each CTA's epilogue drains its own 128
// accumulator rows from its own TMEM. Per SM, a stage then brings in 16 KB of
// W instead of 32 KB for the same tensor-core work.
// Every wait on an mbarrier is bounded; a wait that runs out sets
// DLRM_FLAG_TIMEOUT in the optional status word, ends that role's loop, and
// the CTA still frees its tensor memory and exits.
#include <algorithm>
#include <atomic>
#include <climits>
#include <cstdint>
#include <cstring>

#include <cuda_bf16.h>

#include "dlrm_mlp.h"
#include "launch.h"
#include "tcgen05_common.cuh"

namespace dlrm {
namespace {

constexpr int kLinBM = 128;    // rows of a tile (tcgen05 M)
constexpr int kLinBK = 64;     // K per stage: 64 bf16 = one 128-byte swizzle row
// Shared-memory ring depth: 4 stages, except with 256-column tiles (48 KB
// stages) next to the f32 output staging, where only 3 fit; CTA pairs hold
// half of the W rows per stage (32 KB stages at BN = 256): 6 stages, 5 next
// to the f32 staging. With the three planes of an f32-activation operand in
// one stage (AG = 3: 64 KB stages on pairs, 56 or 64 KB on one CTA at 64 or
// 128 columns), 3 stages, 2 next to the f32 staging at 128 columns or more.
template <int BN, bool F32S, bool PAIR, int AG>
constexpr int lin_stages() {
  if constexpr (PAIR && AG == 3) return F32S ? 2 : 3;
  if constexpr (AG == 3) return (BN >= 128 && F32S) ? 2 : 3;
  if constexpr (PAIR) return F32S ? 5 : 6;
  return (BN >= 256 && F32S) ? 3 : 4;
}
constexpr int kLinEpiWarps = 8;  // two per TMEM lane quarter, each half of the columns
constexpr int kLinThreads = 64 + 32 * kLinEpiWarps;  // producer warp, MMA warp, epilogue
constexpr long long kLinWaitLimit = 200000000LL;  // clock cycles, about 0.1 s
constexpr int kLinMaxDevices = 64;  // devices whose launch set-up is cached

template <int BN, bool F32S, bool PAIR, int AG>
struct LinSmem {
  static constexpr int kStages = lin_stages<BN, F32S, PAIR, AG>();
  static constexpr int kA = kLinBM * kLinBK * 2;
  static constexpr int kB = (PAIR ? BN / 2 : BN) * kLinBK * 2;
  static constexpr int kStage = AG * kA + kB;  // AG A-plane boxes, then the W box
  // After the ring: each epilogue warp's output staging (a 32 x 32 f32 tile in
  // the 128-byte swizzled layout when F32S -- the f32 output goes out through
  // TMA --, then a 32 x 32 bf16 tile in the 64-byte swizzled layout), the
  // bias region (4 BN floats: the whole bias vector, or each warp's slice of
  // the tile's), then the barriers full[S], empty[S], acc_full[2],
  // acc_empty[2], mma_done and the TMEM slot.
  static constexpr int kStage32 = F32S ? 32 * 32 * 4 : 0;
  static constexpr int kStage16 = 32 * 32 * 2;
  static constexpr int kStaging = kStages * kStage;
  static constexpr int kBias = kStaging + kLinEpiWarps * (kStage32 + kStage16);
  static constexpr int kBars = kBias + kLinEpiWarps * (BN / 2) * 4;
  static constexpr int kTotal = kBars + (2 * kStages + 5) * 8 + 8 + 1024;  // + alignment
  static_assert(kTotal <= 227 * 1024, "shared memory of one CTA");
};

// Tensor maps of one launch: the A operand's parts (up to two, lo and hi)
// times their bf16 planes (up to three), the weight planes (up to three), and
// the two TMA-stored outputs.
constexpr int kLinMaxAMaps = 6;
constexpr int kLinMaxWMaps = 3;
constexpr int kLinMaxSegs = 12;
struct alignas(64) LinMaps {
  CUtensorMap a[kLinMaxAMaps];
  CUtensorMap w[kLinMaxWMaps];
  CUtensorMap y32, y16;
  CUtensorMap yp[3];  // the three bf16 planes of an f32-activation output
};

// The K blocks of a tile, in order, are the concatenation of segments: nkb
// blocks of A map `a` from column a_k0 times W map `w` from column w_k0. A
// plain layer is one segment, the split form two (A_lo, then A_hi against W's
// columns k_lo..), and an f32-activation layer one per (A plane, W plane)
// product it sums -- or, when a stage holds all three A planes (AG = 3), one
// per A part, with maps a .. a+2 read against the one W block.
struct LinSeg {
  int a, w, a_k0, w_k0, nkb;
};

struct LinearArgs {
  const float* bias;
  float* y_f32;
  uint16_t* y_bf16;
  uint16_t* y_planes;  // three bf16 planes of the f32 result (exact split), or null
  int64_t ldy_f32, ldy_bf16, ldy_planes, splane_y;
  int M, N;
  LinSeg seg[kLinMaxSegs];
  int nseg, nkb;
  int tiles_n, tiles;  // column tiles; tiles (CTA pairs: 256-row tile pairs)
  int tma_f32, tma_bf16;  // write that output through TMA stores (see the launcher)
  int tma_planes;         // the same for the three planes (through the bf16 staging)
  int32_t* status;
};

template <int ACT>
__device__ __forceinline__ float activate(float x) {
  if constexpr (ACT == DLRM_ACT_RELU) {
    return x > 0.f ? x : 0.f;
  } else if constexpr (ACT == DLRM_ACT_SIGMOID) {
    return __fdiv_rn(1.f, __fadd_rn(1.f, expf(-x)));
  } else {
    return x;
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(lo))) |
         (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(hi))) << 16);
}

// Exact split of an f32 value into three bf16 values, x = p0 + p1 + p2: p0 is x
// with the low 16 bits of its encoding cleared (its top 8 significant bits),
// p1 the same of the remainder x - p0, and p2 = x - p0 - p1, whose at most 8
// significant bits fit a bf16 exactly. Both subtractions are exact.
__device__ __forceinline__ void split_bf16x3(float x, uint16_t& p0, uint16_t& p1, uint16_t& p2) {
  const uint32_t u = __float_as_uint(x);
  const float h0 = __uint_as_float(u & 0xffff0000u);
  const float r = __fsub_rn(x, h0);
  const uint32_t v = __float_as_uint(r);
  const float h1 = __uint_as_float(v & 0xffff0000u);
  const float t = __fsub_rn(r, h1);
  p0 = static_cast<uint16_t>(u >> 16);
  p1 = static_cast<uint16_t>(v >> 16);
  p2 = static_cast<uint16_t>(__float_as_uint(t) >> 16);
}

// Where the epilogue's direct stores go (outputs not written through TMA).
struct LinOut {
  float* y_f32;
  uint16_t* y_bf16;
  uint16_t* y_planes;
  int64_t ldy_f32, ldy_bf16, ldy_planes, splane_y;
  int M, N;
};

// Store 32 consecutive results of one row (columns nb .. nb+31, clipped to N).
__device__ __forceinline__ void store_chunk32(const LinOut& o, int row, int nb,
                                              const float (&v)[32], bool f32_vec, bool bf_vec,
                                              bool planes_vec) {
  if (row >= o.M) return;
  const bool whole = nb + 32 <= o.N;
  if (o.y_f32 != nullptr) {
    float* y = o.y_f32 + static_cast<int64_t>(row) * o.ldy_f32 + nb;
    if (whole && f32_vec) {
#pragma unroll
      for (int q = 0; q < 8; ++q)
        reinterpret_cast<float4*>(y)[q] =
            make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (nb + j < o.N) y[j] = v[j];
    }
  }
  if (o.y_planes != nullptr) {
    uint16_t* y0 = o.y_planes + static_cast<int64_t>(row) * o.ldy_planes + nb;
    uint16_t* y1 = y0 + o.splane_y;
    uint16_t* y2 = y1 + o.splane_y;
    if (whole && planes_vec) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t a[4], b[4], c[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          uint16_t a0, a1, b0, b1, c0, c1;
          split_bf16x3(v[8 * q + 2 * e], a0, b0, c0);
          split_bf16x3(v[8 * q + 2 * e + 1], a1, b1, c1);
          a[e] = a0 | (static_cast<uint32_t>(a1) << 16);
          b[e] = b0 | (static_cast<uint32_t>(b1) << 16);
          c[e] = c0 | (static_cast<uint32_t>(c1) << 16);
        }
        reinterpret_cast<uint4*>(y0)[q] = make_uint4(a[0], a[1], a[2], a[3]);
        reinterpret_cast<uint4*>(y1)[q] = make_uint4(b[0], b[1], b[2], b[3]);
        reinterpret_cast<uint4*>(y2)[q] = make_uint4(c[0], c[1], c[2], c[3]);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (nb + j < o.N) split_bf16x3(v[j], y0[j], y1[j], y2[j]);
    }
  }
  if (o.y_bf16 != nullptr) {
    uint16_t* y = o.y_bf16 + static_cast<int64_t>(row) * o.ldy_bf16 + nb;
    if (whole && bf_vec) {
#pragma unroll
      for (int q = 0; q < 4; ++q)
        reinterpret_cast<uint4*>(y)[q] = make_uint4(
            pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
            pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (nb + j < o.N) y[j] = __bfloat16_as_ushort(__float2bfloat16_rn(v[j]));
    }
  }
}

template <int BN, int ACT, bool F32S, bool PAIR, int AG>
__global__ void __launch_bounds__(kLinThreads, 1)
    linear_bf16_kernel(const __grid_constant__ LinMaps maps, const __grid_constant__ LinearArgs args) {
  using L = LinSmem<BN, F32S, PAIR, AG>;
  constexpr int CG = PAIR ? 2 : 1;
  constexpr int kUnitM = CG * kLinBM;  // rows of the tile a CTA (pair) owns
  constexpr uint32_t kCols = 2 * BN;  // two f32 accumulators (a power of two >= 128)
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);  // 1024-byte aligned tiles
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* empty = full + L::kStages;
  uint64_t* acc_full = empty + L::kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(mma_done + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // CTA pairs: rank in the pair (0 = the MMA issuer), pair index and count
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const int unit0 = PAIR ? static_cast<int>(cluster_id_x()) : static_cast<int>(blockIdx.x);
  const int unit_step = PAIR ? static_cast<int>(cluster_count_x()) : static_cast<int>(gridDim.x);

  if (warp == 1) {
    tmem_alloc<CG>(tslot, kCols);
    tmem_relinquish<CG>();
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      // one arrival per epilogue warp (of both CTAs of a pair: the issuer's
      // barrier gathers them)
      mbar_init(&acc_empty[b], CG * kLinEpiWarps);
    }
    mbar_init(mma_done, 1);
    mbar_init_fence();
  }
  tc_fence_before_sync();
  if constexpr (PAIR)
    cluster_sync();  // both CTAs' barriers exist before either signals the other's
  else
    __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tslot;
  const int nkb = args.nkb;
  // A dependent kernel may be scheduled now; it waits for this grid's results
  // before reading them (griddepcontrol.wait above), and its CTAs only take an
  // SM once one of these has left it.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  bool timed_out = false;

  if (warp == 0) {
    if (lane == 0) {
      // TMA producer: a continuous K-block stream over this CTA's tiles. A may
      // be the previous kernel's output: with programmatic dependent launch
      // this kernel can start while that one finishes, so wait for it here
      // (a no-op without such a dependency).
      asm volatile("griddepcontrol.wait;" ::: "memory");
      int g = 0;
      for (int t = unit0; t < args.tiles && !timed_out; t += unit_step) {
        const int m0 = (t / args.tiles_n) * kUnitM + static_cast<int>(rank) * kLinBM;
        const int n0 = (t % args.tiles_n) * BN;
        int si = 0, sb0 = 0;  // current segment and its first K block
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int s = g % L::kStages;
          if (g >= L::kStages &&
              !mbar_wait_bounded(&empty[s], ((g / L::kStages) - 1) & 1, kLinWaitLimit)) {
            timed_out = true;
            break;
          }
          while (kb - sb0 >= args.seg[si].nkb) sb0 += args.seg[si++].nkb;
          const LinSeg& sg = args.seg[si];
          const int kk = (kb - sb0) * kLinBK;
          uint8_t* sa = smem + s * L::kStage;
          uint8_t* sb = sa + AG * L::kA;
          if constexpr (PAIR) {
            // every stage's bytes (both CTAs') are counted on the issuer's full
            // barrier, which only the issuer's producer arms
            if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * L::kStage);
            const uint32_t fb = map_to_cta(smem_u32(&full[s]), 0);
#pragma unroll
            for (int i = 0; i < AG; ++i)
              tma_load_2d_pair(sa + i * L::kA, &maps.a[sg.a + i], fb, sg.a_k0 + kk, m0);
            tma_load_2d_pair(sb, &maps.w[sg.w], fb, sg.w_k0 + kk,
                             n0 + static_cast<int>(rank) * (BN / 2));
          } else {
            mbar_arrive_expect_tx(&full[s], L::kStage);
#pragma unroll
            for (int i = 0; i < AG; ++i)
              tma_load_2d(sa + i * L::kA, &maps.a[sg.a + i], &full[s], sg.a_k0 + kk, m0);
            tma_load_2d(sb, &maps.w[sg.w], &full[s], sg.w_k0 + kk, n0);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // MMA issuer (of a pair: the even CTA).
      constexpr uint32_t idesc = idesc_bf16_f32(kUnitM, BN);
      int g = 0, j = 0;
      for (int t = unit0; t < args.tiles && !timed_out; t += unit_step, ++j) {
        const int b = j & 1;
        if (j >= 2) {
          const uint32_t par = ((j >> 1) - 1) & 1;
          const bool ok = mbar_wait_bounded(&acc_empty[b], par, kLinWaitLimit);
          if (!ok) {
            timed_out = true;
            break;
          }
        }
        tc_fence_after_sync();
        const uint32_t acc = tmem + static_cast<uint32_t>(b * BN);
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int s = g % L::kStages;
          if (!mbar_wait_bounded(&full[s], (g / L::kStages) & 1, kLinWaitLimit)) {
            timed_out = true;
            break;
          }
          tc_fence_after_sync();
          const uint32_t sa = smem_u32(smem + s * L::kStage);
          const uint32_t sb = sa + AG * L::kA;
#pragma unroll
          for (int i = 0; i < AG; ++i)
#pragma unroll
            for (int kk = 0; kk < kLinBK / 16; ++kk)
              tc_mma_bf16<CG>(acc, sdesc_k_sw128(sa + i * L::kA + kk * 32),
                              sdesc_k_sw128(sb + kk * 32), idesc, (kb | i | kk) != 0 ? 1u : 0u);
          // the stage (both CTAs' halves) is free once these MMAs have read it
          if constexpr (PAIR)
            tc_commit_pair_both(&empty[s]);
          else
            tc_commit<CG>(&empty[s]);
        }
        // the accumulator (both CTAs' rows) is final once all of them are done
        if constexpr (PAIR)
          tc_commit_pair_both(&acc_full[b]);
        else
          tc_commit<CG>(&acc_full[b]);
      }
      // every MMA issued has completed (and read the peer's shared memory)
      // before this CTA or its peer can leave
      tc_commit<CG>(mma_done);
      if (!mbar_wait_bounded(mma_done, 0, kLinWaitLimit)) timed_out = true;
    }
  } else {
    // Epilogue warps 2..9: warp w reads TMEM lane quarter w % 4 (rows 32*(w%4) ..
    // +31 of a tile) and column half (w - 2) / 4 of the accumulator, 32 columns
    // per tcgen05.ld; the bias is read from shared memory (staged below).
    // A 32 x 32 result block goes out either through the warp's staging tiles
    // and one TMA store per output (lane r writes row r; 16-byte chunk q of a row
    // sits at chunk q ^ (r & 7) of a 128-byte f32 row and q ^ ((r >> 1) & 3) of a
    // 64-byte bf16 row, the layouts the maps' 128- and 64-byte swizzles read, so
    // the 32 lanes' 16-byte writes spread over all banks), or with direct stores.
    constexpr int kColsPerWarp = BN / 2;
    const int ew = warp - 2;
    const int quarter = warp & 3;
    const int c_begin = (ew >> 2) * kColsPerWarp;
    float* bias_s = reinterpret_cast<float*>(smem + L::kBias) + ew * kColsPerWarp;
    uint8_t* st32 = smem + L::kStaging + ew * (L::kStage32 + L::kStage16);
    uint8_t* st16 = st32 + L::kStage32;
    const bool f32_vec = args.y_f32 != nullptr && (args.ldy_f32 % 4) == 0 &&
                         (reinterpret_cast<uintptr_t>(args.y_f32) % 16) == 0;
    const bool bf_vec = args.y_bf16 != nullptr && (args.ldy_bf16 % 8) == 0 &&
                        (reinterpret_cast<uintptr_t>(args.y_bf16) % 16) == 0;
    const bool planes_vec = args.y_planes != nullptr && (args.ldy_planes % 8) == 0 &&
                            (args.splane_y % 8) == 0 &&
                            (reinterpret_cast<uintptr_t>(args.y_planes) % 16) == 0;
    const bool tma_out = args.tma_f32 || args.tma_bf16 || args.tma_planes;
    // the outputs not written through TMA
    LinOut direct;
    direct.y_f32 = args.tma_f32 ? nullptr : args.y_f32;
    direct.y_bf16 = args.tma_bf16 ? nullptr : args.y_bf16;
    direct.y_planes = args.tma_planes ? nullptr : args.y_planes;
    direct.ldy_f32 = args.ldy_f32;
    direct.ldy_bf16 = args.ldy_bf16;
    direct.ldy_planes = args.ldy_planes;
    direct.splane_y = args.splane_y;
    direct.M = args.M;
    direct.N = args.N;
    const bool any_direct =
        direct.y_f32 != nullptr || direct.y_bf16 != nullptr || direct.y_planes != nullptr;
    // A bias vector that fits the bias region whole (N <= 4 BN, every layer of
    // the DLRMv1 MLPs) is staged once, by all epilogue warps, zero-filled to a
    // multiple of 32 columns; a longer one is staged per tile, each warp its
    // own slice. (Restaging per tile cost every warp an L2 round trip per tile:
    // with the ring taking the shared memory, L1 keeps no lines across tiles.)
    constexpr int kBiasCols = kLinEpiWarps * kColsPerWarp;
    const bool bias_whole = args.N <= kBiasCols;
    float* bias_all = reinterpret_cast<float*>(smem + L::kBias);
    if (bias_whole) {
      const int n_end = (args.N + 31) & ~31;
      for (int n = ew * 32 + lane; n < n_end; n += kLinEpiWarps * 32)
        bias_all[n] = (args.bias != nullptr && n < args.N) ? __ldg(args.bias + n) : 0.f;
      asm volatile("bar.sync 1, %0;" ::"r"(kLinEpiWarps * 32) : "memory");  // epilogue warps only
    }
    int j = 0;
    for (int t = unit0; t < args.tiles; t += unit_step, ++j) {
      const int b = j & 1;
      const int m0 = (t / args.tiles_n) * kUnitM + static_cast<int>(rank) * kLinBM;
      const int n0 = (t % args.tiles_n) * BN;
      const float* bias_w = bias_whole ? bias_all + n0 + c_begin : bias_s;  // column c_begin
      if (!bias_whole) {
        for (int c = lane; c < kColsPerWarp; c += 32) {
          const int n = n0 + c_begin + c;
          bias_s[c] = (args.bias != nullptr && n < args.N) ? __ldg(args.bias + n) : 0.f;
        }
        __syncwarp();
      }
      const bool ok =
          __all_sync(0xffffffffu, mbar_wait_bounded(&acc_full[b], (j >> 1) & 1, kLinWaitLimit));
      if (!ok) {
        timed_out = true;
        break;
      }
      tc_fence_after_sync();
      const int row0 = m0 + quarter * 32;
      const uint32_t trow =
          tmem + static_cast<uint32_t>(b * BN) + (static_cast<uint32_t>(quarter * 32) << 16);
#pragma unroll 1
      for (int c0 = c_begin; c0 < c_begin + kColsPerWarp && n0 + c0 < args.N; c0 += 32) {
        float v[32];
        tmem_ld_32x32b_x32(trow + c0, v);
        const float4* bq = reinterpret_cast<const float4*>(bias_w + (c0 - c_begin));
        if (ACT != DLRM_ACT_SIGMOID || n0 + c0 + 32 <= args.N) {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 bb = bq[q];
            v[4 * q] = activate<ACT>(__fadd_rn(v[4 * q], bb.x));
            v[4 * q + 1] = activate<ACT>(__fadd_rn(v[4 * q + 1], bb.y));
            v[4 * q + 2] = activate<ACT>(__fadd_rn(v[4 * q + 2], bb.z));
            v[4 * q + 3] = activate<ACT>(__fadd_rn(v[4 * q + 3], bb.w));
          }
        } else {
          // the sigmoid of the columns past N (never stored) is skipped: the
          // 256 -> 1 output layer would evaluate 32 of them for one
          const float* bs = reinterpret_cast<const float*>(bq);
          const int valid = args.N - (n0 + c0);  // 1 .. 31, the same in every lane
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i < valid) v[i] = activate<ACT>(__fadd_rn(v[i], bs[i]));
        }
        if (tma_out) {
          if (lane == 0) bulk_wait_read_all();  // the previous block has left the staging
          __syncwarp();
          if (F32S && args.tma_f32) {
            uint4* rowp = reinterpret_cast<uint4*>(st32 + lane * 128);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              rowp[q ^ (lane & 7)] =
                  make_uint4(__float_as_uint(v[4 * q]), __float_as_uint(v[4 * q + 1]),
                             __float_as_uint(v[4 * q + 2]), __float_as_uint(v[4 * q + 3]));
          }
          if (args.tma_bf16) {
            uint4* rowp = reinterpret_cast<uint4*>(st16 + lane * 64);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              rowp[q ^ ((lane >> 1) & 3)] = make_uint4(
                  pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                  pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (F32S && args.tma_f32) tma_store_2d(&maps.y32, st32, n0 + c0, row0);
            if (args.tma_bf16) tma_store_2d(&maps.y16, st16, n0 + c0, row0);
            bulk_commit();
          }
          if (args.tma_planes) {
            // the three planes one after another through the bf16 staging tile
            // (an f32-activation layer writes no bf16 output)
#pragma unroll
            for (int p = 0; p < 3; ++p) {
              if (p > 0) {
                if (lane == 0) bulk_wait_read_all();  // the previous plane has left
                __syncwarp();
              }
              uint4* rowp = reinterpret_cast<uint4*>(st16 + lane * 64);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                uint32_t w4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  uint32_t h[2];
#pragma unroll
                  for (int u = 0; u < 2; ++u) {
                    uint16_t a0, a1, a2;
                    split_bf16x3(v[8 * q + 2 * e + u], a0, a1, a2);
                    h[u] = p == 0 ? a0 : (p == 1 ? a1 : a2);
                  }
                  w4[e] = h[0] | (h[1] << 16);
                }
                rowp[q ^ ((lane >> 1) & 3)] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
              }
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_2d(&maps.yp[p], st16, n0 + c0, row0);
                bulk_commit();
              }
            }
          }
        }
        if (any_direct) store_chunk32(direct, row0 + lane, n0 + c0, v, f32_vec, bf_vec, planes_vec);
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) {  // this warp has drained its share
        if constexpr (PAIR)  // on the issuer's barrier, for both CTAs' warps
          mbar_arrive_remote(map_to_cta(smem_u32(&acc_empty[b]), 0));
        else
          mbar_arrive(&acc_empty[b]);
      }
    }
    if (lane == 0) bulk_wait_all();  // every TMA store of this warp has completed
  }
  if (timed_out && args.status != nullptr) atomicOr(args.status, DLRM_FLAG_TIMEOUT);
  tc_fence_before_sync();
  if constexpr (PAIR)
    cluster_sync();  // neither CTA leaves while the other may still use its memory
  else
    __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc<CG>(tmem, kCols);
}

__global__ void f32_to_bf16_kernel(const float* __restrict__ x, int64_t ldx, int64_t rows,
                                   int64_t cols, uint16_t* __restrict__ y, int64_t ldy) {
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const float* xr = x + r * ldx;
    uint16_t* yr = y + r * ldy;
    for (int64_t c = threadIdx.x; c < cols; c += blockDim.x)
      yr[c] = __bfloat16_as_ushort(__float2bfloat16_rn(__ldg(xr + c)));
  }
}

// 2-D bf16 tensor map {cols, rows} with row pitch ld elements, box {64, box_rows},
// 128-byte swizzle; elements past the tensor read as zero.
cudaError_t encode_bf16_operand(CUtensorMap* map, const void* base, int64_t cols, int64_t rows,
                                int64_t ld, int box_rows) {
  const EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kLinBK), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int BN, int ACT, bool F32S, bool PAIR, int AG>
cudaError_t run_linear(const LinMaps& maps, LinearArgs args, int sms, cudaStream_t stream) {
  auto* fn = &linear_bf16_kernel<BN, ACT, F32S, PAIR, AG>;
  constexpr int smem = LinSmem<BN, F32S, PAIR, AG>::kTotal;
  constexpr int kUnitM = (PAIR ? 2 : 1) * kLinBM;
  // Per device, the instance's shared-memory size is set and (pairs) the
  // resident cluster count queried once: 0 = not yet, else that count + 1.
  // Both are fixed for a device and an instance, so later launches skip the
  // two driver calls.
  static std::atomic<int> prepared[kLinMaxDevices];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    dev = -1;
  }
  const bool cacheable = dev >= 0 && dev < kLinMaxDevices;
  const int cached = cacheable ? prepared[dev].load(std::memory_order_acquire) : 0;
  cudaError_t e = cudaSuccess;
  if (cached == 0) {
    e = cudaFuncSetAttribute(reinterpret_cast<const void*>(fn),
                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
  }
  int fit = cached > 0 ? cached - 1 : 0;
  args.tiles_n = (args.N + BN - 1) / BN;
  const int64_t tiles = static_cast<int64_t>((args.M + kUnitM - 1) / kUnitM) * args.tiles_n;
  if (tiles > INT32_MAX) return cudaErrorInvalidValue;
  args.tiles = static_cast<int>(tiles);
  // programmatic dependent launch: the prologue (TMEM allocation, barriers)
  // overlaps the tail of the kernel before it on the stream
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kLinThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // one CTA per SM: the shared-memory ring and the 2 x BN TMEM columns size it
  int64_t grid = std::min<int64_t>(tiles, sms);
  if constexpr (PAIR) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
    // as many pairs as can be resident at once (a GPC with an odd number of
    // free SMs leaves one idle)
    int pairs = sms / 2;
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
    if (cached == 0 && cudaOccupancyMaxActiveClusters(&fit, fn, &cfg) != cudaSuccess) {
      (void)cudaGetLastError();
      fit = 0;
    }
    if (fit > 0) pairs = std::min(pairs, fit);
    grid = 2 * std::min<int64_t>(tiles, pairs);
  }
  if (cacheable && cached == 0) prepared[dev].store(fit + 1, std::memory_order_release);
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  return cudaLaunchKernelEx(&cfg, fn, maps, args);
}

template <int BN, bool F32S, bool PAIR, int AG>
cudaError_t run_linear_act(int act, const LinMaps& maps, const LinearArgs& args, int sms,
                           cudaStream_t stream) {
  switch (act) {
    case DLRM_ACT_RELU:
      return run_linear<BN, DLRM_ACT_RELU, F32S, PAIR, AG>(maps, args, sms, stream);
    case DLRM_ACT_SIGMOID:
      return run_linear<BN, DLRM_ACT_SIGMOID, F32S, PAIR, AG>(maps, args, sms, stream);
    default: return run_linear<BN, DLRM_ACT_NONE, F32S, PAIR, AG>(maps, args, sms, stream);
  }
}

// The instance with f32 output staging (and, at 256 columns on one CTA, a
// 3-stage ring) only when the f32 output goes out through TMA.
template <int BN, bool PAIR = false, int AG = 1>
cudaError_t run_linear_bn(int act, const LinMaps& maps, const LinearArgs& args, int sms,
                          cudaStream_t stream) {
  return args.tma_f32 ? run_linear_act<BN, true, PAIR, AG>(act, maps, args, sms, stream)
                      : run_linear_act<BN, false, PAIR, AG>(act, maps, args, sms, stream);
}

// 2-D output map {N, M} with row pitch ld elements, box {32, 32}, written from a
// staging tile in the given swizzle layout.
cudaError_t encode_output(CUtensorMap* map, void* base, CUtensorMapDataType dt, int esz, int64_t N,
                          int64_t M, int64_t ld, CUtensorMapSwizzle swz) {
  const EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * esz};
  const cuuint32_t box[2] = {32, 32};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, dt, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         swz, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

int sm_count_current() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n;
}

// Tile width: the widest of 256, 128 whose tile count still covers every SM,
// else 64 (more, smaller tiles for small layers).
int choose_bn(int64_t M, int64_t N, int sms) {
#ifdef DLRM_LIN_FORCE_BN
  if (N > 64) return DLRM_LIN_FORCE_BN;
#endif
  const int64_t mt = (M + kLinBM - 1) / kLinBM;
  if (N <= 64) return 64;
  if (mt * ((N + 255) / 256) >= sms) return 256;
  if (mt * ((N + 127) / 128) >= sms) return 128;
  return 64;
}

// 256-column tiles run on CTA pairs (256 x 256 per pair) when the pairs' tile
// count still covers every SM. Measured on B200 at B=65536 against one CTA per
// tile: f32 activations, 3, 24 and 30 K blocks per tile, 58.4 -> 54.3 us,
// 67.6 -> 63.0 us and 124.4 -> 106.6 us; bf16 activations, 1, 8 and 10 K
// blocks, 35.7 -> 33.8 us, 31.7 -> 29.7 us and 50.1 -> 45.0 us.
bool choose_pair(int64_t M, int64_t N, int bn, int sms) {
#ifdef DLRM_LIN_NO_PAIR
  return false;
#endif
  return bn == 256 &&
         ((M + 2 * kLinBM - 1) / (2 * kLinBM)) * ((N + 255) / 256) >= sms / 2;
}

bool is_aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }


// One layer: the checks shared by both entry points are done; `parts` lists
// the A parts (1 or 2) as (base, pitch, plane stride, k) with `a_planes`
// planes each, W has `w_planes` planes. Builds the maps and the segment table
// and launches.
struct APart {
  const uint16_t* base;
  int64_t ld, splane, k;
};

int launch_layer(const APart* parts, int nparts, int a_planes, const uint16_t* w, int64_t ldw,
                 int64_t splane_w, int w_planes, const float* bias, int64_t M, int64_t N,
                 int act, float* y_f32, int64_t ldy_f32, uint16_t* y_bf16, int64_t ldy_bf16,
                 uint16_t* y_planes, int64_t ldy_planes, int64_t splane_y, int32_t* status_dev,
                 cudaStream_t stream) {
  const int64_t K = parts[0].k + (nparts > 1 ? parts[1].k : 0);
  const int sms = sm_count_current();
  const int bn = choose_bn(M, N, sms);
  const bool pair = choose_pair(M, N, bn, sms);
  LinMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  cudaError_t e = cudaSuccess;
  for (int p = 0; p < nparts && e == cudaSuccess; ++p)
    for (int i = 0; i < a_planes && e == cudaSuccess; ++i)
      e = encode_bf16_operand(&maps.a[p * 3 + i], parts[p].base + i * parts[p].splane,
                              parts[p].k, M, parts[p].ld, kLinBM);
  for (int j = 0; j < w_planes && e == cudaSuccess; ++j)
    e = encode_bf16_operand(&maps.w[j], w + j * splane_w, K, N, ldw, pair ? bn / 2 : bn);
  if (e != cudaSuccess) return cuda_fail(e);

  LinearArgs args;
  std::memset(&args, 0, sizeof(args));
  args.bias = bias;
  args.y_f32 = y_f32;
  args.y_bf16 = y_bf16;
  args.y_planes = y_planes;
  args.ldy_f32 = ldy_f32;
  args.ldy_bf16 = ldy_bf16;
  args.ldy_planes = ldy_planes;
  args.splane_y = splane_y;
  args.M = static_cast<int>(M);
  args.N = static_cast<int>(N);
  args.status = status_dev;
  // Products summed: A plane i times W plane j for i + j < 3 (all three A
  // planes against a single weight plane; against three weight planes the six
  // products whose planes' leading bits lie within 2^-16 of the value's).
  // Three A planes against one weight plane load the planes into one stage
  // next to the W block they share (AG = 3): a third of the W bytes per tile.
  // Not at 256 columns on one CTA (an 80 KB stage leaves too shallow a ring).
  // Measured on B200 (f32 activations, bf16 weights): at B=65536 top layer 0
  // (pairs, 30 K blocks per tile) 106.5 -> 98.3 us, the 13 -> 512 layer 53.3 ->
  // 49.1 us, the 64-column layers 34.8 -> 30.7 us; at B=2048 (one CTA per
  // tile) every layer 1.5-3 us faster, the f32 forward graph 112.6 -> 101.6 us.
  const bool group_planes = a_planes == 3 && w_planes == 1 && (pair || bn <= 128);
  int w_off = 0;
  for (int p = 0; p < nparts && group_planes; ++p) {
    const int nkb = static_cast<int>((parts[p].k + kLinBK - 1) / kLinBK);
    LinSeg& sg = args.seg[args.nseg++];
    sg.a = p * 3;
    sg.w = 0;
    sg.a_k0 = 0;
    sg.w_k0 = w_off;
    sg.nkb = nkb;
    args.nkb += nkb;
    w_off += static_cast<int>(parts[p].k);
  }
  for (int p = 0; p < nparts && !group_planes; ++p) {
    const int nkb = static_cast<int>((parts[p].k + kLinBK - 1) / kLinBK);
    for (int i = 0; i < a_planes; ++i)
      for (int j = 0; j < w_planes; ++j) {
        if (i + j >= 3) continue;
        LinSeg& sg = args.seg[args.nseg++];
        sg.a = p * 3 + i;
        sg.w = j;
        sg.a_k0 = 0;
        sg.w_k0 = w_off;
        sg.nkb = nkb;
        args.nkb += nkb;
      }
    w_off += static_cast<int>(parts[p].k);
  }
  // Outputs whose rows are whole 16-byte units at 16-byte aligned addresses go
  // out through TMA stores; the others are written directly.
  args.tma_f32 = y_f32 != nullptr && ldy_f32 % 4 == 0 && is_aligned(y_f32, 16);
  args.tma_bf16 = y_bf16 != nullptr && ldy_bf16 % 8 == 0 && is_aligned(y_bf16, 16);
  if (args.tma_f32)
    e = encode_output(&maps.y32, y_f32, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, N, M, ldy_f32,
                      CU_TENSOR_MAP_SWIZZLE_128B);
  if (e == cudaSuccess && args.tma_bf16)
    e = encode_output(&maps.y16, y_bf16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N, M, ldy_bf16,
                      CU_TENSOR_MAP_SWIZZLE_64B);
  // the planes go out through the bf16 staging tile, which a layer writing
  // planes does not otherwise use
  args.tma_planes = y_planes != nullptr && y_bf16 == nullptr && ldy_planes % 8 == 0 &&
                    splane_y % 8 == 0 && is_aligned(y_planes, 16);
  for (int p = 0; p < 3 && e == cudaSuccess && args.tma_planes; ++p)
    e = encode_output(&maps.yp[p], y_planes + p * splane_y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, N,
                      M, ldy_planes, CU_TENSOR_MAP_SWIZZLE_64B);
  if (e != cudaSuccess) return cuda_fail(e);
  switch (bn) {
    case 256:
      e = !pair         ? run_linear_bn<256>(act, maps, args, sms, stream)
          : group_planes ? run_linear_bn<256, true, 3>(act, maps, args, sms, stream)
                         : run_linear_bn<256, true>(act, maps, args, sms, stream);
      break;
    case 128:
      e = group_planes ? run_linear_bn<128, false, 3>(act, maps, args, sms, stream)
                       : run_linear_bn<128>(act, maps, args, sms, stream);
      break;
    default:
      e = group_planes ? run_linear_bn<64, false, 3>(act, maps, args, sms, stream)
                       : run_linear_bn<64>(act, maps, args, sms, stream);
      break;
  }
  if (e != cudaSuccess) return cuda_fail(e);
  note_launch();
  return DLRM_OK;
}

// Shape and alignment checks of one layer (see dlrm_mlp.h).
int check_layer(const APart* parts, int nparts, const uint16_t* w, int64_t ldw,
                const float* bias, int64_t M, int64_t N, int act, const float* y_f32,
                int64_t ldy_f32, const uint16_t* y_bf16, int64_t ldy_bf16,
                const uint16_t* y_planes, int64_t ldy_planes, const int32_t* status_dev) {
  if (parts[0].base == nullptr || w == nullptr) return DLRM_ERR_NULL;
  if (y_f32 == nullptr && y_bf16 == nullptr && y_planes == nullptr) return DLRM_ERR_NULL;
  if (nparts > 1 && parts[1].base == nullptr) return DLRM_ERR_NULL;
  if (act < DLRM_ACT_NONE || act > DLRM_ACT_SIGMOID) return DLRM_ERR_ARG;
  if (M < 1 || N < 1 || parts[0].k < 1 || (nparts > 1 && parts[1].k < 1)) return DLRM_ERR_SHAPE;
  const int64_t K = parts[0].k + (nparts > 1 ? parts[1].k : 0);
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return DLRM_ERR_SHAPE;
  for (int p = 0; p < nparts; ++p)
    if (parts[p].ld < parts[p].k) return DLRM_ERR_SHAPE;
  if (ldw < K) return DLRM_ERR_SHAPE;
  if ((y_f32 != nullptr && ldy_f32 < N) || (y_bf16 != nullptr && ldy_bf16 < N) ||
      (y_planes != nullptr && ldy_planes < N))
    return DLRM_ERR_SHAPE;
  if ((N + 63) / 64 > 65535) return DLRM_ERR_SHAPE;
  for (int p = 0; p < nparts; ++p)
    if (parts[p].ld % 8 != 0 || !is_aligned(parts[p].base, 16)) return DLRM_ERR_ALIGN;
  if (ldw % 8 != 0 || !is_aligned(w, 16)) return DLRM_ERR_ALIGN;
  if (nparts > 1 && parts[0].k % 8 != 0) return DLRM_ERR_ALIGN;
  if ((bias != nullptr && !is_aligned(bias, 4)) || (y_f32 != nullptr && !is_aligned(y_f32, 4)) ||
      (y_bf16 != nullptr && !is_aligned(y_bf16, 2)) ||
      (y_planes != nullptr && !is_aligned(y_planes, 2)) ||
      (status_dev != nullptr && !is_aligned(status_dev, 4)))
    return DLRM_ERR_ALIGN;
  return DLRM_OK;
}

__global__ void split_bf16x3_kernel(const float* __restrict__ x, int64_t ldx, int64_t rows,
                                    int64_t cols, uint16_t* __restrict__ y, int64_t ldy,
                                    int64_t splane) {
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const float* xr = x + r * ldx;
    uint16_t* yr = y + r * ldy;
    for (int64_t c = threadIdx.x; c < cols; c += blockDim.x)
      split_bf16x3(__ldg(xr + c), yr[c], yr[c + splane], yr[c + 2 * splane]);
  }
}

}  // namespace
}  // namespace dlrm

extern "C" {

DLRM_API int dlrm_linear_bf16(const uint16_t* a_lo, int64_t lda_lo, int64_t k_lo,
                              const uint16_t* a_hi, int64_t lda_hi, int64_t k_hi,
                              const uint16_t* w, int64_t ldw, const float* bias, int64_t M,
                              int64_t N, int act, float* y_f32, int64_t ldy_f32,
                              uint16_t* y_bf16, int64_t ldy_bf16, int32_t* status_dev,
                              dlrm_stream_t stream) {
  using namespace dlrm;
  if (k_hi < 0) return DLRM_ERR_SHAPE;
  const APart parts[2] = {{a_lo, lda_lo, 0, k_lo}, {a_hi, lda_hi, 0, k_hi}};
  const int nparts = k_hi > 0 ? 2 : 1;
  int rc = check_layer(parts, nparts, w, ldw, bias, M, N, act, y_f32, ldy_f32, y_bf16, ldy_bf16,
                       nullptr, 0, status_dev);
  if (rc != DLRM_OK) return rc;
  return launch_layer(parts, nparts, 1, w, ldw, 0, 1, bias, M, N, act, y_f32, ldy_f32, y_bf16,
                      ldy_bf16, nullptr, 0, 0, status_dev,
                      reinterpret_cast<cudaStream_t>(stream));
}

DLRM_API int dlrm_linear_f32a(const uint16_t* a_lo, int64_t lda_lo, int64_t splane_lo,
                              int64_t k_lo, const uint16_t* a_hi, int64_t lda_hi,
                              int64_t splane_hi, int64_t k_hi, const uint16_t* w, int64_t ldw,
                              int64_t splane_w, int w_planes, const float* bias, int64_t M,
                              int64_t N, int act, float* y_f32, int64_t ldy_f32,
                              uint16_t* y_planes, int64_t ldy_planes, int64_t splane_y,
                              int32_t* status_dev, dlrm_stream_t stream) {
  using namespace dlrm;
  if (k_hi < 0) return DLRM_ERR_SHAPE;
  if (w_planes != 1 && w_planes != 3) return DLRM_ERR_ARG;
  const APart parts[2] = {{a_lo, lda_lo, splane_lo, k_lo}, {a_hi, lda_hi, splane_hi, k_hi}};
  const int nparts = k_hi > 0 ? 2 : 1;
  int rc = check_layer(parts, nparts, w, ldw, bias, M, N, act, y_f32, ldy_f32, nullptr, 0,
                       y_planes, ldy_planes, status_dev);
  if (rc != DLRM_OK) return rc;
  // plane strides: whole 16-byte rows apart, and the planes must not overlap
  for (int p = 0; p < nparts; ++p)
    if (parts[p].splane % 8 != 0) return DLRM_ERR_ALIGN;
  if (w_planes == 3 && splane_w % 8 != 0) return DLRM_ERR_ALIGN;
  if (splane_lo < (M - 1) * lda_lo + k_lo || (k_hi > 0 && splane_hi < (M - 1) * lda_hi + k_hi) ||
      (w_planes == 3 && splane_w < (N - 1) * ldw + k_lo + k_hi) ||
      (y_planes != nullptr && splane_y < (M - 1) * ldy_planes + N))
    return DLRM_ERR_SHAPE;
  return launch_layer(parts, nparts, 3, w, ldw, splane_w, w_planes, bias, M, N, act, y_f32,
                      ldy_f32, nullptr, 0, y_planes, ldy_planes, splane_y, status_dev,
                      reinterpret_cast<cudaStream_t>(stream));
}

DLRM_API int dlrm_split_f32_bf16x3(const float* x, int64_t ldx, int64_t rows, int64_t cols,
                                   uint16_t* y, int64_t ldy, int64_t splane,
                                   dlrm_stream_t stream) {
  using namespace dlrm;
  if (x == nullptr || y == nullptr) return DLRM_ERR_NULL;
  if (rows < 1 || cols < 1 || ldx < cols || ldy < cols) return DLRM_ERR_SHAPE;
  if (splane < (rows - 1) * ldy + cols) return DLRM_ERR_SHAPE;
  if (!is_aligned(x, 4) || !is_aligned(y, 2)) return DLRM_ERR_ALIGN;
  const int64_t blocks = std::min<int64_t>(rows, 148 * 32);
  const int threads = cols >= 256 ? 256 : static_cast<int>(((cols + 31) / 32) * 32);
  split_bf16x3_kernel<<<static_cast<unsigned>(blocks), threads, 0,
                        reinterpret_cast<cudaStream_t>(stream)>>>(x, ldx, rows, cols, y, ldy,
                                                                 splane);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  note_launch();
  return DLRM_OK;
}

DLRM_API int dlrm_f32_to_bf16(const float* x, int64_t ldx, int64_t rows, int64_t cols,
                              uint16_t* y, int64_t ldy, dlrm_stream_t stream) {
  using namespace dlrm;
  if (x == nullptr || y == nullptr) return DLRM_ERR_NULL;
  if (rows < 1 || cols < 1 || ldx < cols || ldy < cols) return DLRM_ERR_SHAPE;
  if (!is_aligned(x, 4) || !is_aligned(y, 2)) return DLRM_ERR_ALIGN;
  const int64_t blocks = std::min<int64_t>(rows, 148 * 32);
  const int threads = cols >= 256 ? 256 : static_cast<int>(((cols + 31) / 32) * 32);
  f32_to_bf16_kernel<<<static_cast<unsigned>(blocks), threads, 0,
                       reinterpret_cast<cudaStream_t>(stream)>>>(x, ldx, rows, cols, y, ldy);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  note_launch();
  return DLRM_OK;
}

}  // extern "C"
