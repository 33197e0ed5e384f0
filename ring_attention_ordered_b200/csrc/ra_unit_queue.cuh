// The work queue of a persistent launch (sm_100a).
//
// The CTAs of a launch take work units from one atomic counter, in the order
// of the unit index (the kernels number their units longest first, so the
// causal load balance of "Ring Attention 环注意力", L4 §4.5, limitation 3,
// comes from the counter itself).  Inside a CTA the loader warp takes the
// next unit and publishes it to the CTA's other roles through
// UNIT_QUEUE_DEPTH shared-memory slots; slot k % depth carries the CTA's
// k-th unit and has an mbarrier (one arrival) that completes once per use.
// A published -1 means that the launch has no more units.
//
// The depth must exceed how far the loader can run ahead of the slowest
// reader: a slot is written again only after every reader has taken the unit
// it held before.  Each kernel states its bound where it uses the queue.
#pragma once

#include <cstdint>

#include "ptx_sm100.cuh"
#include "ra_sync.cuh"

namespace ra {

constexpr int UNIT_QUEUE_DEPTH = 4;

struct UnitQueue {
  uint32_t bar0;    // UNIT_QUEUE_DEPTH mbarriers, 8 bytes apart (shared address)
  uint32_t slots;   // UNIT_QUEUE_DEPTH ints (shared address)

  __device__ __forceinline__ uint32_t bar(int k) const {
    return bar0 + 8u * static_cast<uint32_t>(k % UNIT_QUEUE_DEPTH);
  }
  __device__ __forceinline__ uint32_t slot(int k) const {
    return slots + 4u * static_cast<uint32_t>(k % UNIT_QUEUE_DEPTH);
  }
  // One thread, before the CTA-wide barrier that precedes the roles.
  __device__ __forceinline__ void init() const {
    for (int i = 0; i < UNIT_QUEUE_DEPTH; ++i) mbar_init(bar0 + 8u * i, 1);
  }
  // Loader warp, all lanes: take the CTA's k-th unit from the launch's
  // counter (-1 once all `total` units are handed out) and publish it.
  // Returns the unit, the same on every lane.
  __device__ __forceinline__ int take(unsigned int* tickets, int total, int k) const {
    int u = 0;
    if ((threadIdx.x & 31) == 0) {
      const unsigned t = atomicAdd(tickets, 1u);
      u = t < static_cast<unsigned>(total) ? static_cast<int>(t) : -1;
      asm volatile("st.shared.s32 [%0], %1;" ::"r"(slot(k)), "r"(u) : "memory");
      mbar_arrive(bar(k));
    }
    return __shfl_sync(0xffffffffu, u, 0);
  }
  // Any other warp, all lanes: the CTA's k-th unit (bounded wait).  Returns
  // false if the kernel is aborting; `u` is the same on every lane.
  __device__ __forceinline__ bool read(int k, const Ctl& cx, uint32_t site, int& u) const {
    const bool ok = wait_bar(bar(k), static_cast<uint32_t>(k / UNIT_QUEUE_DEPTH) & 1u, cx, site);
    if (!__all_sync(0xffffffffu, ok)) return false;
    asm volatile("ld.shared.s32 %0, [%1];" : "=r"(u) : "r"(slot(k)) : "memory");
    u = __shfl_sync(0xffffffffu, u, 0);
    return true;
  }
};

}  // namespace ra
