// Bounded wait on a count in global memory, for kernels whose CTAs hand work
// to each other within one launch (all CTAs resident at once).
#pragma once

#include "sm100_ptx.cuh"

namespace engram {
namespace sm100 {

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Wait until *p >= target, for at most kWaitLimitNs (then raise the CTA's
// abort flag and kDevErrTimeout).  The reads have acquire semantics: what the
// counting threads made visible before their increments is visible after the
// wait returns true.
static __device__ __noinline__ bool wait_count(const unsigned* p, unsigned target,
                                               volatile int* abort_flag, unsigned* err) {
  const uint64_t t0 = globaltimer();
  while (ld_acquire_u32(p) < target) {
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicOr(err, kDevErrTimeout);
      return false;
    }
    __nanosleep(32);
  }
  return true;
}

}  // namespace sm100
}  // namespace engram
