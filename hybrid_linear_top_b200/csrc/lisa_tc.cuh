// Thin wrappers over the sm_100a tensor-core (tcgen05) instructions used by
// the prefill contractions: TMEM allocation, MMA from shared-memory
// descriptors into a TMEM accumulator, commit to an mbarrier, TMEM loads.
#pragma once

#include "lisa_common.cuh"

namespace lisa {

// ---------------------------------------------------------------- TMEM allocation (one full warp)
__device__ __forceinline__ void tc_alloc(uint32_t *dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// ---------------------------------------------------------------- ordering
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Makes this thread's generic-proxy shared-memory writes visible to the
// tensor core (async proxy).
__device__ __forceinline__ void fence_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- descriptors
// Instruction descriptor, kind::f16: bf16 A and B, fp32 D, M x N; A / B
// K-major unless a_mn / b_mn (then MN-major).
__host__ __device__ constexpr uint32_t tc_idesc_bf16(int M, int N, bool a_mn = false, bool b_mn = false) {
  return (1u << 4)                       // D format: f32
         | (1u << 7)                     // A format: bf16
         | (1u << 10)                    // B format: bf16
         | ((a_mn ? 1u : 0u) << 15)      // A major
         | ((b_mn ? 1u : 0u) << 16)      // B major
         | ((uint32_t)(N >> 3) << 17)    // N / 8
         | ((uint32_t)(M >> 4) << 24);   // M / 16
}

// Shared-memory matrix descriptor of an MN-major operand with a 128-byte
// swizzle: each 128-byte row holds 64 consecutive M (or N) elements of one K
// index, 8 rows form a 1024-byte group (groups 1024 bytes apart), and the
// next 64 M / N elements start `lbo_bytes` further.  +2048 bytes = +16 in K.
__device__ __forceinline__ uint64_t tc_sdesc_mnmajor(uint32_t smem_addr, uint32_t lbo_bytes) {
  const uint64_t start = (smem_addr & 0x3FFFFu) >> 4;
  return start | ((uint64_t)(lbo_bytes >> 4) << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

// Byte offset of element (row, col) of a [rows][128] bf16 tile stored as two
// 128-byte-swizzled halves of 64 columns (`half_bytes` apart) -- the layout
// TMA writes with a {64, rows} box and the 128-byte swizzle.
__device__ __forceinline__ uint32_t sw128_offset(int row, int col, uint32_t half_bytes) {
  const int half = col >> 6, cc = col & 63;
  return (uint32_t)half * half_bytes + (uint32_t)(row >> 3) * 1024u + (uint32_t)(row & 7) * 128u +
         (uint32_t)((((cc >> 3) ^ (row & 7)) << 4) + (cc & 7) * 2);
}

// Shared-memory matrix descriptor of a K-major operand whose rows are
// `row_bytes` (128 or 64) long and swizzled in 16-byte chunks by TMA with the
// matching swizzle span; the tile starts at a 1024-byte (128) / 512-byte (64)
// aligned address; 8-row groups are 8 * row_bytes apart.
__device__ __forceinline__ uint64_t tc_sdesc_kmajor(uint32_t smem_addr, int row_bytes) {
  const uint64_t start = (smem_addr & 0x3FFFFu) >> 4;
  const uint64_t lbo = 1;                                   // unused by the swizzled K-major forms
  const uint64_t sbo = (uint64_t)(8 * row_bytes) >> 4;
  const uint64_t layout = row_bytes == 128 ? 2u : 4u;       // SWIZZLE_128B : SWIZZLE_64B
  return start | (lbo << 16) | (sbo << 32) | (1ull << 46) | (layout << 61);
}

// ---------------------------------------------------------------- MMA and commit (one thread)
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrives once on `bar` when every tcgen05.mma this thread issued before has completed.
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// ---------------------------------------------------------------- TMEM -> registers (one full warp)
// 32 lanes x 32 bits, 16 consecutive columns: thread i gets lane (base + i), columns [col, col+16).
__device__ __forceinline__ void tc_ld16(uint32_t taddr, uint32_t *r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tc_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 4-D tiled TMA load, coordinates from the innermost.
__device__ __forceinline__ void tma_load_4d(void *dst, const void *tmap, int c0, int c1, int c2, int c3,
                                            uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, "
      "%5}], [%6];" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
      : "memory");
}

// 3-D tiled TMA load, coordinates {innermost, middle, outer}.
__device__ __forceinline__ void tma_load_3d(void *dst, const void *tmap, int c0, int c1, int c2, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

}  // namespace lisa
