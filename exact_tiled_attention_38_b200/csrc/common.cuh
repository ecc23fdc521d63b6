// Device status word and bounded mbarrier waits shared by the kernels.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace eta {

// First device-side error wins; the host reads and clears it. Codes are
// kStatusTimeout | site, where site says which wait gave up.
__device__ unsigned int g_status = 0;

constexpr unsigned kStatusTimeout = 0x1000u;
constexpr uint64_t kDefaultWaitNs = 2000000000ull;  // 2 s: every real wait is microseconds

// Per-CTA control block in shared memory.
struct CtaCtl {
  int abort;          // set once any wait in the CTA gives up
  int pad;
  uint64_t wait_ns;   // time limit of one wait
};

__device__ __forceinline__ void record_status(unsigned code) { atomicCAS(&g_status, 0u, code); }

__device__ __noinline__ bool wait_slow(uint32_t bar, uint32_t parity, CtaCtl* ctl, unsigned site,
                                       bool honour_abort) {
  const uint64_t t0 = globaltimer_ns();
  volatile int* abort = &ctl->abort;
  for (uint32_t n = 1;; ++n) {
    if (mbar_try_wait_sleep(bar, parity)) return true;
    if ((n & 15u) == 0) {
      if (honour_abort && *abort) return false;
      if (globaltimer_ns() - t0 > ctl->wait_ns) {
        *abort = 1;
        record_status(kStatusTimeout | site);
        return false;
      }
    }
  }
}

// Wait until the phase with the given parity of `bar` has completed. Returns
// false (without completing) when the CTA is aborting or the time limit passed.
// The first poll sleeps in try_wait with a suspend-time hint, so a waiting
// thread takes no issue slots from its neighbours and is woken as soon as the
// phase completes; only if that poll times out does the wait read the global
// timer (a slow read) and start checking the time limit.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, CtaCtl* ctl,
                                         unsigned site) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait_sleep(a, parity)) return true;
  return wait_slow(a, parity, ctl, site, true);
}

// Same, but keeps waiting (up to the limit) even when the CTA aborts: used to
// drain copies or MMAs still in flight before the CTA exits.
__device__ __forceinline__ bool drain_bar(uint64_t* bar, uint32_t parity, CtaCtl* ctl,
                                          unsigned site) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  return wait_slow(a, parity, ctl, site, false);
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

}  // namespace eta
