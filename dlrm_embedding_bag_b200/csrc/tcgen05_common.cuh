// Inline-PTX wrappers for the 5th-generation tensor cores of sm_100a used by
// the MLP layers: tensor-memory (TMEM) allocation, the single-thread
// tcgen05.mma issue with shared-memory matrix descriptors, tcgen05.commit onto
// an mbarrier, tcgen05.ld of the f32 accumulator, and the 2-D TMA tile load
// that stages the operands.
//
// CG is the CTA group of the tcgen05 operations: 1 (one CTA, M = 128 per
// MMA) or 2 (a CTA pair of a cluster, M = 256 per MMA: the pair's even CTA
// issues the MMA, each CTA holds half of A's rows and half of B's rows in its
// shared memory at the same offsets, and each CTA's TMEM receives its own 128
// rows of D). A kernel uses one CTA group for all of its tcgen05 operations.
//
// No multicast form of any TMA load is used.
#pragma once

#include <cstdint>

#include "tma_common.cuh"

namespace dlrm {

// ---- TMEM ---------------------------------------------------------------

// Allocate `ncols` TMEM columns (a power of two >= 32) for this CTA; the base
// address lands in *dst. Executed by one whole warp (with CG = 2 by one warp
// in each CTA of the pair, which get the same address).
template <int CG = 1>
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  if constexpr (CG == 2)
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
  else
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}

// Give up the right to allocate more (lets other CTAs on the SM allocate).
template <int CG = 1>
__device__ __forceinline__ void tmem_relinquish() {
  if constexpr (CG == 2)
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  else
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

// Free what tmem_alloc returned. Executed by one whole warp (per CTA).
template <int CG = 1>
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  if constexpr (CG == 2)
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
  else
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// Order tcgen05 operations across a thread synchronisation.
__device__ __forceinline__ void tc_fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ---- descriptors ----------------------------------------------------------

// Shared-memory matrix descriptor of a K-major operand tile stored in the
// 128-byte-swizzled layout that a TMA load with CU_TENSOR_MAP_SWIZZLE_128B
// writes: rows of 128 bytes (64 bf16 along K), groups of 8 rows 1024 bytes
// apart. Fields: start address >> 4 (bits 0-13), leading-dimension byte
// offset >> 4 (16-29; unused for swizzled K-major layouts, set to 1), stride
// byte offset >> 4 (32-45; 1024 B between 8-row groups), descriptor version
// 1 (46-47), base offset 0 (49-51; the tile starts on a 1024-byte boundary),
// layout type 2 = 128-byte swizzle (61-63). A K-slice that starts k bytes
// into the 128-byte rows is addressed by adding k to the start address.
__device__ __forceinline__ uint64_t sdesc_k_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(1) << 16;
  d |= static_cast<uint64_t>(1024 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Instruction descriptor of tcgen05.mma.kind::f16 with bf16 A and B, both
// K-major, f32 accumulation, dense, shape M x N: D format F32 (bits 4-5 = 1),
// A format BF16 (7-9 = 1), B format BF16 (10-12 = 1), N >> 3 (17-22),
// M >> 4 (24-28).
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// ---- MMA --------------------------------------------------------------

// D[tmem] (+)= A[smem] * B[smem]^T for one K=16 step; accumulate = 0 starts
// the accumulator from zero. Issued by a single thread (with CG = 2, of the
// pair's even CTA; the descriptors' addresses select the same tiles in both).
template <int CG = 1>
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  if constexpr (CG == 2)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// One arrival on `bar` (this CTA's) once every tcgen05 operation this thread
// issued so far has completed.
template <int CG = 1>
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  if constexpr (CG == 2)
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
  else
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// CTA pair: one arrival on the mbarrier at `bar`'s offset in each CTA of the
// pair (mask 0b11) once every tcgen05 operation this thread issued so far has
// completed. This is the completion signal of the tensor cores, not a copy.
__device__ __forceinline__ void tc_commit_pair_both(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(static_cast<uint16_t>(0x3))
      : "memory");
}

// ---- TMEM -> registers ------------------------------------------------------

// 32 consecutive 32-bit columns of the warp's 32 TMEM lanes (lane i of the
// warp gets row i of its quarter): taddr = base + (32*(warp%4) << 16) + col.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// ---- TMA ------------------------------------------------------------------

// The box of a 2-D tensor map at (x, y) (x innermost, in elements; x * element
// size a multiple of 16 bytes) lands at dst; completion is counted on bar in
// bytes. Out-of-range elements read as zero.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// CTA pair: the box of a 2-D tensor map at (x, y) lands at dst in this CTA's
// shared memory; completion is counted in bytes on the mbarrier at the
// shared::cluster address `bar_cluster`, which may be the peer CTA's (the even
// CTA's barrier counts both CTAs' tiles of a stage). Not a multicast load.
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map,
                                                 uint32_t bar_cluster, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}

// The box at (x, y) of a 2-D tensor map is written from src (shared memory,
// laid out as the map's swizzle mode dictates); elements outside the tensor are
// not written. Completion is tracked by bulk async-groups (commit / wait below).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int x,
                                             int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until this thread's committed bulk stores have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until this thread's committed bulk stores have completed.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

}  // namespace dlrm
