// Building blocks of the fifth-generation tensor cores (sm_100a, tcgen05):
// tensor-memory allocation, shared-memory matrix descriptors, the f16 MMA
// with an fp32 accumulator in tensor memory, commit to an mbarrier, and the
// 32-lane tensor-memory loads of the epilogue.
//
// Operand layout used here (both operands K-major, no swizzle): a tile of R
// rows x 64 columns of fp16 is stored as 8 column chunks of 16 bytes, chunk c
// of row r at byte c*(R*16) + r*16. In the descriptor's terms that is the
// canonical interleaved K-major form: rows of one 8-row core matrix 16 bytes
// apart, successive 8-row groups 128 bytes apart (stride byte offset), the two
// 16-byte column chunks an MMA of K = 16 reads R*16 bytes apart (leading byte
// offset). One MMA takes K = 16, i.e. chunks 2s and 2s+1 of the tile.
#pragma once

#include <stdint.h>

#include "common.cuh"

namespace qmoe {

// ------------------------------------------------------------------ descriptors
// Shared-memory matrix descriptor (no swizzle): start address, leading byte
// offset (K direction), stride byte offset (M/N direction), all >> 4;
// descriptor version 1 in bits 46-47, layout type 0 (no swizzle) in 61-63.
__device__ __forceinline__ uint64_t tc_smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  return d;
}
// Instruction descriptor of kind::f16: fp32 accumulator (bits 4-5 = 1), A and
// B fp16 (formats 0), both K-major, N >> 3 in bits 17-22, M >> 4 in bits 24-28.
__host__ __device__ constexpr uint32_t tc_idesc_f16(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ------------------------------------------------------------------ tensor memory
// One warp: allocates `ncols` columns (a power of two >= 32) and writes the
// base address to *slot (shared memory).
__device__ __forceinline__ void tc_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               :: "r"(smem_u32(slot)), "r"(ncols) : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// ------------------------------------------------------------------ MMA (one thread issues)
// D[tmem] (+)= A * B^T, A M x 16 and B N x 16 from shared memory (descriptors).
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           bool accumulate) {
  const uint32_t acc = accumulate ? 1u : 0u, z = 0u;
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n}\n"
      :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc), "r"(z) : "memory");
}
// The mbarrier receives one arrival when every MMA this thread issued before
// has completed (and its shared-memory operands may be overwritten).
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               :: "r"(smem_u32(bar)) : "memory");
}

// ------------------------------------------------------------------ epilogue loads
// Warp w of a warpgroup reads tensor-memory lanes 32(w%4) .. 32(w%4)+31: thread
// i gets lane 32(w%4)+i, 16 consecutive 32-bit columns from `taddr`.
__device__ __forceinline__ void tc_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

}  // namespace qmoe
