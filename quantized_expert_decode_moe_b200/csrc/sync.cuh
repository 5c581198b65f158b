// Synchronisation building blocks of the decode kernels (sm_100a): shared-memory
// mbarriers completed by bulk copies, and a grid-wide barrier on counters in the
// workspace header. Every wait is bounded by %globaltimer; a wait that runs out
// latches MOE_ERR_TIMEOUT in the status word and returns false.
#pragma once

#include "common.cuh"

namespace qmoe {

// ------------------------------------------------------------------ mbarrier and bulk copies
__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
// orders this thread's earlier generic-proxy accesses of shared memory before its later bulk copies
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}
// global -> shared bulk copy of `bytes` (multiple of 16; both addresses 16-byte aligned), counted on bar
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void latch_timeout(uint32_t* status) {
  if (status) atomicCAS(status, 0u, (uint32_t)MOE_ERR_TIMEOUT);
}
// Waits for the phase of parity `parity` of bar, for at most bound_ns; on
// timeout latches MOE_ERR_TIMEOUT in *status and returns false.
static __device__ __noinline__ bool mbar_wait_slow(uint64_t* bar, unsigned parity, unsigned long long bound_ns,
                                            uint32_t* status) {
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > bound_ns) {
      latch_timeout(status);
      return false;
    }
  }
  return true;
}
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, unsigned parity, unsigned long long bound_ns,
                                                  uint32_t* status) {
  return mbar_try_wait(bar, parity) || mbar_wait_slow(bar, parity, bound_ns, status);
}

// ------------------------------------------------------------------ grid-wide barrier
// One barrier = an arrival counter and a generation word in global memory
// (the workspace header). A round: every CTA of the grid arrives once; the
// last arrival resets the counter to 0 and then advances the generation; a
// CTA waits until the generation differs from the value it read before it
// arrived. The counter is 0 between rounds, so the grid size may change from
// one launch to the next, and arrival and wait may be split (arrive early,
// wait much later). A CTA reads the generation before arriving; the round
// cannot complete before its own arrival, so the value read is the one the
// round will advance.
//
// Ordering: the CTA's threads finish their global writes, __syncthreads(),
// then one thread calls grid_arrive (fence, then the atomic: release of the
// whole CTA's writes). The waiting thread's acquire load, followed by
// __syncthreads(), orders the CTA's later loads after every arrival's writes.
// Data produced by other CTAs is read with L1-bypassing loads (__ldcg).
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_u32(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}

struct GridBar {
  unsigned* cnt;   // arrivals of the current round
  unsigned* gen;   // generation (rounds completed, mod 2^32)
};

// One thread per CTA. Returns the generation the round will advance.
__device__ __forceinline__ unsigned grid_arrive(GridBar b, unsigned nctas) {
  const unsigned g = ld_acquire_u32(b.gen);
  __threadfence();
  const unsigned old = atomicAdd(b.cnt, 1u);
  if (old == nctas - 1) {
    *(volatile unsigned*)b.cnt = 0u;
    __threadfence();
    st_release_u32(b.gen, g + 1u);
  }
  return g;
}
// One thread per CTA: waits (at most bound_ns) for the round of generation g
// to complete; on timeout latches MOE_ERR_TIMEOUT and returns false.
static __device__ __noinline__ bool grid_wait(GridBar b, unsigned g, unsigned long long bound_ns, uint32_t* status) {
  if (ld_acquire_u32(b.gen) != g) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (ld_acquire_u32(b.gen) == g) {
    if (globaltimer_ns() - t0 > bound_ns) {
      latch_timeout(status);
      return false;
    }
  }
  return true;
}

}  // namespace qmoe
