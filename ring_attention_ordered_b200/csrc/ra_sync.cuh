// Bounded mbarrier waits shared by the kernels (sm_100a).
//
// Every wait gives up after a time limit (%globaltimer): it then records
// RA_ERR_TIMEOUT with the wait site and CTA in the kernel's device status
// word, raises the CTA's shared abort flag (every other wait of the CTA
// checks it) and returns false, so the roles drain what they have in flight,
// free their tensor memory and return instead of hanging the GPU.
#pragma once

#include <cstdint>

#include "ptx_sm100.cuh"
#include "ring_attn.h"

// Longest single hardware suspension inside one mbarrier try_wait (ns).
#ifndef RA_WAIT_HINT_NS
#define RA_WAIT_HINT_NS 1000000u
#endif

namespace ra {

struct Ctl {
  volatile uint32_t* abort;
  unsigned long long limit_ns;
  unsigned long long* status;   // the kernel's device status word
};

static __device__ __noinline__ void record_timeout(const Ctl& cx, uint32_t site) {
  *cx.abort = 1u;
  const unsigned long long code =
      (static_cast<unsigned long long>(RA_ERR_TIMEOUT) << 32) | (site << 16) | (blockIdx.x & 0xFFFF);
  atomicCAS(cx.status, 0ull, code);
}

// Bounded wait on an mbarrier phase.  Returns false if the kernel is aborting
// (this wait ran out, or another role's did).
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, const Ctl& cx,
                                         uint32_t site) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity, RA_WAIT_HINT_NS)) return true;
    if (*cx.abort) return false;
    if (globaltimer_ns() - t0 > cx.limit_ns) {
      record_timeout(cx, site);
      return false;
    }
  }
}

// Short bounded wait used only while draining after an abort.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > ns) return;
  }
}

// Bounded wait executed by a whole warp; the result is warp-uniform.
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, const Ctl& cx,
                                          uint32_t site) {
  const bool ok = wait_bar(bar, parity, cx, site);
  return __all_sync(0xffffffffu, ok);
}

}  // namespace ra
