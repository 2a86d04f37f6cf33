// tc_util.cuh -- sm_100a tensor-core building blocks written as inline PTX:
// tiled TMA loads (no multicast), tcgen05 TMEM allocation, MMA issue,
// commit-to-mbarrier, TMEM loads, and the shared-memory / instruction
// descriptors of tcgen05.mma kind::f16.
//
// Descriptor formats (sm_100 UMMA, as laid out in CUTLASS's
// cute/arch/mma_sm100_desc.hpp):
//   shared-memory descriptor (64 bit): start address >> 4 [0,14), leading
//   byte offset >> 4 [16,30), stride byte offset >> 4 [32,46), version = 1
//   [46,48), base offset [49,52), LBO mode [52], layout type [61,64)
//   (2 = 128-byte swizzle).
//   instruction descriptor (32 bit): D format [4,6) (1 = f32), A format
//   [7,10) and B format [10,13) (1 = bf16), A major [15], B major [16]
//   (0 = K-major, 1 = MN-major), N >> 3 [17,23), M >> 4 [24,29).
//   An MN-major operand tile is read through the same descriptor format as
//   desc_mnmajor_sw128 below (64-element MN blocks `leading byte offset`
//   apart, 8-row K groups 1024 B apart).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "async_util.cuh"

namespace sfn {

// ---------------------------------------------------------------- TMA
// 2-D tiled load of box {c0 .. c0+box0, c1 .. c1+box1} into shared memory,
// completing on `bar`.  c0 (innermost, elements) must be a multiple of 8 for
// 16-bit elements; the callers only use multiples of 64.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int c0, int c1,
                                            uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// As tma_load_2d, with an L2 eviction-priority policy (make_evict_first_policy
// for data read once).
__device__ __forceinline__ void tma_load_2d_hint(void *dst, const CUtensorMap *map, int c0, int c1,
                                                 uint64_t *bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- TMEM
// Allocate `ncols` (power of two >= 32) TMEM columns; the base address is
// written to *slot (shared memory).  Executed by one whole warp.
__device__ __forceinline__ void tmem_alloc(uint32_t *slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(slot)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t base, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 in, f32 accumulate).
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once all previously issued tcgen05.mma of this thread are
// complete (and their shared-memory operands may be overwritten).
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread (lane) gets its row's 32
// values.  taddr = tmem base + (lane_base << 16) + column.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
        "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
        "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
        "=r"(v[31])
      : "r"(taddr));
}
// As tmem_ld_32x32b_x32, 16 consecutive columns.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
        "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------- descriptors
// K-major operand tile, rows of 64 bf16 (128 B) written by TMA with the
// 128-byte swizzle; 8-row groups 1024 B apart.  Advance along K by 16
// elements = +32 bytes of start address.
__device__ __forceinline__ uint64_t desc_kmajor_sw128(const void *smem_tile) {
  const uint32_t a = smem_u32(smem_tile);
  return (uint64_t)((a >> 4) & 0x3fffu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// MN-major operand tile: TMA boxes of 64 (MN) x 64 (K) bf16, each box a
// column of 64 K-rows of 128 bytes (64 MN-elements) with the 128-byte
// swizzle; consecutive 64-element MN blocks are `mn_block_bytes` apart
// (leading byte offset), 8-row K groups 1024 B apart (stride byte offset).
// Advance along K by 16 rows = +2048 bytes of start address.
__device__ __forceinline__ uint64_t desc_mnmajor_sw128(const void *smem_tile,
                                                       uint32_t mn_block_bytes) {
  const uint32_t a = smem_u32(smem_tile);
  return (uint64_t)((a >> 4) & 0x3fffu) | ((uint64_t)((mn_block_bytes >> 4) & 0x3fffu) << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor: bf16 x bf16 -> f32, M x N, A and B each K- or
// MN-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool b_mn_major,
                                                      bool a_mn_major = false) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) |
         ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// Host: the driver's tensor-map encoder (false if unavailable), and a
// row-major bf16 matrix [outer][inner] (rows `stride` elements apart, 0:
// inner) as a 2-D map with box {box_inner, box_outer}, 128-byte swizzle and
// zero fill outside the matrix.
bool encoder();
bool make_map(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer,
              uint32_t box_inner, uint32_t box_outer, uint64_t stride = 0);

}  // namespace sfn
