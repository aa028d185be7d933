// Fifth-generation tensor-core helpers of sm_100a (tcgen05): shared-memory
// matrix descriptors, the instruction descriptor of kind::f16 with f32
// accumulation, tensor-memory (TMEM) allocation, the MMA itself, its commit to
// an mbarrier and the TMEM -> register loads. Hand-written PTX.
//
// Layout conventions used by every caller:
//  * operands are K-major with the 128-byte swizzle, i.e. exactly what a 2-D
//    tensor copy with a 64 x rows fp16 box and CU_TENSOR_MAP_SWIZZLE_128B
//    writes: row r of an atom at r * 128 bytes, its 16-byte chunk c stored at
//    chunk c ^ (r % 8); atoms 1024-byte aligned, 8-row groups 1024 bytes apart;
//  * one MMA consumes K = 16 fp16 (32 bytes of a row); the next K step of the
//    same atom starts 32 bytes further (the swizzle is applied by the
//    hardware on the absolute address, so the start address simply advances);
//  * the accumulator of an M = 128 MMA is 128 TMEM lanes (row i of D in lane
//    i) by N columns of 32 bits; warp w of the CTA may only read lanes
//    32 * (w % 4) ... + 31.
#pragma once

#include <stdint.h>

#include "tq_common.cuh"

namespace tq {

// Shared-memory descriptor of a K-major, 128-byte-swizzled operand whose
// first row starts at shared address `addr` (16-byte units in bits 0-13;
// leading offset 1 (unused by swizzled K-major layouts); stride between
// 8-row groups 1024 bytes; descriptor version 1; swizzle mode 2 = 128 B).
TQ_DEV uint64_t umma_desc_sw128(uint32_t addr) {
  uint64_t d = (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

// Instruction descriptor of tcgen05.mma kind::f16: fp16 A and B (both
// K-major), f32 accumulator, M x N tile.
__host__ __device__ constexpr uint32_t umma_idesc_f16(int M, int N) {
  return (1u << 4)                       // D format: f32
         | (0u << 7) | (0u << 10)        // A, B format: f16
         | ((uint32_t)(N >> 3) << 17)    // N / 8
         | ((uint32_t)(M >> 4) << 24);   // M / 16
}

// ---------------------------------------------------------------- TMEM allocation
// Executed by one whole warp. The base address (lane 0, first column) is
// written to shared memory at `dst`.
TQ_DEV void tmem_alloc(uint32_t dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst), "r"(ncols)
               : "memory");
}
TQ_DEV void tmem_relinquish() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory"); }
TQ_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// ---------------------------------------------------------------- ordering
TQ_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
TQ_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// ---------------------------------------------------------------- MMA
// D[tmem] (+)= A[adesc] * B[bdesc]^T, issued by a single thread.
TQ_DEV void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"((uint32_t)accumulate)
      : "memory");
}

// Arrive once on the mbarrier when every tcgen05 operation issued so far by
// this thread has completed (no multicast).
TQ_DEV void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// ---------------------------------------------------------------- TMEM -> registers
// Thread t of the warp reads lane (lane field of taddr) + t, N consecutive
// 32-bit columns starting at the column field of taddr.
TQ_DEV void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
TQ_DEV void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}
TQ_DEV void tmem_ld4(uint32_t taddr, uint32_t (&r)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr));
}
TQ_DEV void tmem_ld2(uint32_t taddr, uint32_t (&r)[2]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(taddr));
}
TQ_DEV void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// The registers written by tcgen05.ld hold valid data only after
// tcgen05.wait::ld; passing them through an empty volatile asm placed after
// the wait makes every later use depend on it, so the compiler cannot hoist
// a use above the wait.
template <int N>
TQ_DEV void tmem_regs_after_wait(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

}  // namespace tq
