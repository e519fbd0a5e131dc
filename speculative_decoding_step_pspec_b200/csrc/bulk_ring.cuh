// bulk_ring.cuh -- per-warp rings of shared-memory stages filled by bulk asynchronous copies
// (sm_90+ `cp.async.bulk`, completion counted in bytes on an mbarrier).
//
// A warp streams a contiguous run of one or two rows through kStages stages of its own:
// lane 0 starts the copy of a chunk into a free stage, every lane waits on the stage's
// mbarrier, reads the chunk from shared memory, and after a __syncwarp lane 0 refills the
// stage with the chunk kStages ahead.  The bytes in flight no longer sit in registers, so a
// CTA keeps tens of kilobytes of loads outstanding at any register budget.
//
// Every wait is bounded: after kRingSpinLimit unsuccessful polls the waiter reports failure
// and its caller sets an error bit and stops issuing copies.
#pragma once

#include <stdint.h>

namespace pspec {

constexpr unsigned kRingSpinLimit = 1u << 21;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// One arrival expected per phase (lane 0's arrive.expect_tx); the copies' bytes complete it.
__device__ __forceinline__ void mbar_init(uint64_t* bar) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(bar)) : "memory");
}

// Makes the initialised barriers visible to the copy engine.
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

// Orders this thread's earlier generic-proxy accesses of shared memory (the reads of the
// stage being refilled, made visible to it by __syncwarp) before the copy that overwrites it.
__device__ __forceinline__ void fence_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Global -> this CTA's shared memory, `bytes` a multiple of 16, both addresses 16-byte aligned.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, unsigned bytes,
                                              uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Waits for the phase of parity `parity` to complete; false after `limit` polls.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned parity,
                                          unsigned limit = kRingSpinLimit) {
  const uint32_t a = smem_addr(bar);
  for (unsigned spin = 0; spin < limit; ++spin) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(a), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}

}  // namespace pspec
