// The parts the bf16 and FP8 forward kernels share: the shared-memory
// barrier set, the per-CTA unit queue, the TMA loader role and the MMA role.
// They differ only in tile geometry and MMA kind, which a geometry policy G
// supplies (G::Q_BYTES, G::KV_BYTES, G::NS, G::OFF_Q, G::OFF_KV; G::load_q,
// G::load_kv; the descriptors and G::issue_qk, G::issue_pv_half).  The
// parameter struct P is FwdParams or Fp8FwdParams (same scheduling fields).
//
// Work: a launch's units (two 128-row query tiles that see the same K/V
// stream) are taken from one queue, an atomic counter over units sorted
// longest first (the causal load balance of "Ring Attention 环注意力",
// L4 §4.5, limitation 3); within a unit the K/V tiles follow the ring order
// (L3 definition, L4 §4.2).  Each CTA's loader takes the next unit and
// publishes it to the CTA's MMA warp and softmax warpgroups.
//
// MMA order per K/V tile j: P0 V (first 64 keys as soon as the softmax has
// stored that half of P0, then the rest), S0(j+1), P1 V, S1(j+1): while one
// tile's softmax runs, the tensor core works on the other tile.
#pragma once

#include <cstdint>

#include "ptx_sm100.cuh"
#include "ra_schedule.cuh"
#include "ra_sync.cuh"

namespace ra {

constexpr int FWD_BM = 128;   // query rows per tile
constexpr int FWD_BN = 128;   // keys per K/V tile

enum FwdWaitSite : uint32_t {
  SITE_Q_FULL = 1, SITE_Q_EMPTY, SITE_KV_FULL, SITE_KV_EMPTY, SITE_S_FULL,
  SITE_P_FULL, SITE_O_DONE, SITE_O_FREE, SITE_P_HALF, SITE_UNIT
};

// Depth of the per-CTA unit queue: the loader publishes each unit it takes
// in slot k % UQ; the MMA warp and the softmax warpgroups read it there.
// The loader can be at most two units ahead of the softmax warpgroups (it
// starts unit k + 1 only after the MMA warp has finished unit k's Q K^T,
// which needs unit k - 1's P), so four slots never overrun.
constexpr int UQ = 4;

// Barriers: q_full, q_empty, kv_full[NS], kv_empty[NS], s_full[2],
// p_full[2], o_done[2], o_free[2], p_half[2], drain, unit_full[UQ].
__host__ __device__ constexpr int fwd_num_bars(int ns) { return 2 + 2 * ns + 10 + 1 + UQ; }

struct FwdBars {
  uint32_t q_full, q_empty, kv_full0, kv_empty0, s_full0, p_full0, o_done0, o_free0, p_half0,
      drain, unit_full0;
  uint32_t units;   // shared address of the unit queue (UQ ints)
  __device__ __forceinline__ uint32_t kv_full(int s) const { return kv_full0 + 8u * s; }
  __device__ __forceinline__ uint32_t kv_empty(int s) const { return kv_empty0 + 8u * s; }
  __device__ __forceinline__ uint32_t s_full(int w) const { return s_full0 + 8u * w; }
  __device__ __forceinline__ uint32_t p_full(int w) const { return p_full0 + 8u * w; }
  __device__ __forceinline__ uint32_t o_done(int w) const { return o_done0 + 8u * w; }
  __device__ __forceinline__ uint32_t o_free(int w) const { return o_free0 + 8u * w; }
  __device__ __forceinline__ uint32_t p_half(int w) const { return p_half0 + 8u * w; }
  __device__ __forceinline__ uint32_t unit_full(int k) const { return unit_full0 + 8u * (k % UQ); }

  // Lay the barriers out from `bar0` (8 bytes each) with NS K/V stages and
  // the unit queue at `units_addr`.
  __device__ __forceinline__ void layout(uint32_t bar0, int ns, uint32_t units_addr) {
    q_full = bar0;
    q_empty = q_full + 8;
    kv_full0 = q_empty + 8;
    kv_empty0 = kv_full0 + 8 * ns;
    s_full0 = kv_empty0 + 8 * ns;
    p_full0 = s_full0 + 16;
    o_done0 = p_full0 + 16;
    o_free0 = o_done0 + 16;
    p_half0 = o_free0 + 16;
    drain = p_half0 + 16;
    unit_full0 = drain + 8;
    units = units_addr;
  }

  // Arrival counts (one thread, before the CTA-wide barrier).
  __device__ __forceinline__ void init(int ns) const {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < ns; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(s_full(w), 1);
      mbar_init(p_full(w), 128);
      mbar_init(o_done(w), 1);
      mbar_init(o_free(w), 128);
      mbar_init(p_half(w), 128);
    }
    mbar_init(drain, 1);
    for (int i = 0; i < UQ; ++i) mbar_init(unit_full0 + 8u * i, 1);
  }
};

// The k-th unit this CTA processes, as published by its loader (-1: no more
// units).  Bounded wait; returns false if the kernel is aborting.
__device__ __forceinline__ bool next_unit(const FwdBars& br, int k, const Ctl& cx, int& u) {
  if (!wait_bar(br.unit_full(k), (k / UQ) & 1, cx, SITE_UNIT)) return false;
  asm volatile("ld.shared.s32 %0, [%1];" : "=r"(u) : "r"(br.units + 4u * (k % UQ)) : "memory");
  return true;
}

// ------------------------------------------------------------------ loader
// The whole warp runs the control flow, so every address and coordinate is
// warp-uniform (uniform registers); one elected lane issues the copies.
template <class G, class P>
__device__ void fwd_loader_role(const P& p, const FwdBars& br, uint32_t smem_base, const Ctl& cx) {
  const bool leader = (threadIdx.x & 31) == 0;
  uint32_t kv_it = 0, q_uses = 0;
  bool q_pending = false;
  for (int k = 0;; ++k) {
    // take the next unit of the launch and publish it to this CTA's roles
    int u = 0;
    if (leader) {
      const unsigned t = atomicAdd(p.tickets, 1u);
      u = t < static_cast<unsigned>(p.total_units) ? static_cast<int>(t) : -1;
      asm volatile("st.shared.s32 [%0], %1;" ::"r"(br.units + 4u * (k % UQ)), "r"(u) : "memory");
      mbar_arrive(br.unit_full(k));
    }
    u = __shfl_sync(0xffffffffu, u, 0);
    if (u < 0) break;
    const Unit x = decode_unit(p, u);
    if (q_uses > 0 && !wait_warp(br.q_empty, (q_uses - 1) & 1u, cx, SITE_Q_EMPTY)) goto drain;
    if ((p.debug_flags & 1u) && q_uses == 0) {
      // fault injection: the first query tiles are never requested
    } else {
      const int row0 = x.b * p.L + x.blk * p.blk_len;
      if (elect_one()) {
        mbar_arrive_expect_tx(br.q_full, (x.valid1 ? 2 : 1) * G::Q_BYTES);
        G::load_q(smem_base + G::OFF_Q, &p.tm_q, br.q_full, x.h[0], row0 + x.qt[0] * FWD_BM);
        if (x.valid1)
          G::load_q(smem_base + G::OFF_Q + G::Q_BYTES, &p.tm_q, br.q_full, x.h[1],
                    row0 + x.qt[1] * FWD_BM);
      }
      __syncwarp();
      q_pending = true;
    }
    ++q_uses;
    KvIter it;
    it.start(p, x);
    for (int idx = 0; idx < x.n_kv; ++idx, it.next(p)) {
      const int row = x.b * p.L + it.jb * p.blk_len + it.kl * FWD_BN;
#pragma unroll
      for (int kv = 0; kv < 2; ++kv) {
        const int s = kv_it % G::NS;
        const uint32_t ph = (kv_it / G::NS) & 1u;
        if (!wait_warp(br.kv_empty(s), ph ^ 1u, cx, SITE_KV_EMPTY)) goto drain;
        const CUtensorMap* map = kv ? &p.tm_v : &p.tm_k;
        if (elect_one()) {
          mbar_arrive_expect_tx(br.kv_full(s), G::KV_BYTES);
          G::load_kv(smem_base + G::OFF_KV + s * G::KV_BYTES, map, br.kv_full(s), x.kvh, row);
        }
        __syncwarp();
        ++kv_it;
      }
    }
  }
  return;
drain:
  // Let the copies already issued land before the CTA's shared memory goes.
  if (leader) {
    const uint32_t n = kv_it < static_cast<uint32_t>(G::NS) ? kv_it : G::NS;
    for (uint32_t i = 0; i < n; ++i) {
      const uint32_t it = kv_it - 1 - i;
      drain_wait(br.kv_full(it % G::NS), (it / G::NS) & 1u, 200000000ull);
    }
    if (q_pending) drain_wait(br.q_full, (q_uses - 1) & 1u, 200000000ull);
  }
  __syncwarp();
}

// ------------------------------------------------------------------ MMA
// TMEM: S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512) fp32 columns;
// P_w overwrites the first columns of S_w.  The commit that signals S_w(j+1)
// fires only after P_w V(j), so the softmax may rescale O right after
// reading S.
template <class G, class P>
__device__ void fwd_mma_role(const P& p, const FwdBars& br, uint32_t smem_base, uint32_t tmem,
                             const Ctl& cx) {
  const bool leader = (threadIdx.x & 31) == 0;
  uint32_t kv_it = 0, q_uses = 0;
  uint32_t pf_phase0 = 0u, pf_phase1 = 0u;
  uint32_t units0 = 0u, units1 = 0u;
  const G g(smem_base);
  auto issue_qk = [&](int w, int stage) { g.issue_qk(tmem + w * 128, w, stage); };
  auto issue_pv_half = [&](int w, int stage, int half, bool acc) {
    if (half == 0)
      g.template issue_pv_half<0>(tmem + 256 + w * 128, tmem + w * 128, stage, acc ? 1u : 0u);
    else
      g.template issue_pv_half<1>(tmem + 256 + w * 128, tmem + w * 128, stage, 1u);
  };
  auto commit = [&](uint32_t bar) {
    if (elect_one()) tc_commit(bar);
  };

  for (int k = 0;; ++k) {
    int u;
    if (!next_unit(br, k, cx, u)) goto drain;
    u = __shfl_sync(0xffffffffu, u, 0);
    if (u < 0) break;
    const Unit x = decode_unit(p, u);
    const int n = x.n_kv;
    if (!wait_warp(br.q_full, q_uses & 1u, cx, SITE_Q_FULL)) goto drain;
    tc_fence_after();
    ++q_uses;
    {
      const int ks = kv_it % G::NS;
      if (!wait_warp(br.kv_full(ks), (kv_it / G::NS) & 1u, cx, SITE_KV_FULL)) goto drain;
      tc_fence_after();
      issue_qk(0, ks);
      commit(br.s_full(0));
      if (x.valid1) {
        issue_qk(1, ks);
        commit(br.s_full(1));
      }
      commit(br.kv_empty(ks));
      ++kv_it;
      if (n == 1) commit(br.q_empty);
    }
    // Barrier states probed ahead of time: a probe issued before a batch of
    // MMAs overlaps its latency with their issue, and a barrier found
    // complete is not waited on again.
    bool rdy_v = false, rdy_k = false, rdy_p0 = false;
    for (int idx = 0; idx < n; ++idx) {
      const bool more = idx + 1 < n;
      const int vs = kv_it % G::NS;
      const int ks = (kv_it + 1) % G::NS;
      if (!rdy_v && !wait_warp(br.kv_full(vs), (kv_it / G::NS) & 1u, cx, SITE_KV_FULL)) goto drain;
      // the next K tile is needed right after P0 V: wait for it now, off the
      // softmax -> MMA -> softmax chain
      if (more && !rdy_k &&
          !wait_warp(br.kv_full(ks), ((kv_it + 1) / G::NS) & 1u, cx, SITE_KV_FULL))
        goto drain;
      tc_fence_after();
      // query tile 0: P0 V in two halves as P0 arrives, then S0 for the next
      // K/V tile
      if (idx == 0 && units0 > 0) {
        if (!wait_warp(br.o_free(0), (units0 - 1) & 1u, cx, SITE_O_FREE)) goto drain;
      }
      if (!rdy_p0 && !wait_warp(br.p_half(0), pf_phase0, cx, SITE_P_HALF)) goto drain;
      tc_fence_after();
      issue_pv_half(0, vs, 0, idx > 0);
      if (!wait_warp(br.p_full(0), pf_phase0, cx, SITE_P_FULL)) goto drain;
      pf_phase0 ^= 1u;
      tc_fence_after();
      issue_pv_half(0, vs, 1, true);
      if (!more) commit(br.o_done(0));
      // probe P1's first half now; the vote on the result comes after the
      // S0 MMAs, so the probe's latency overlaps their issue
      const bool raw_p1 = x.valid1 ? mbar_test_wait(br.p_half(1), pf_phase1) : true;
      if (more) {
        issue_qk(0, ks);
        commit(br.s_full(0));
      }
      const bool rdy_p1 = __all_sync(0xffffffffu, raw_p1);
      // query tile 1
      if (x.valid1) {
        if (idx == 0 && units1 > 0) {
          if (!wait_warp(br.o_free(1), (units1 - 1) & 1u, cx, SITE_O_FREE)) goto drain;
        }
        if (!rdy_p1 && !wait_warp(br.p_half(1), pf_phase1, cx, SITE_P_HALF)) goto drain;
        tc_fence_after();
        issue_pv_half(1, vs, 0, idx > 0);
        if (!wait_warp(br.p_full(1), pf_phase1, cx, SITE_P_FULL)) goto drain;
        pf_phase1 ^= 1u;
        tc_fence_after();
        issue_pv_half(1, vs, 1, true);
        if (!more) commit(br.o_done(1));
      }
      // V of this step has been read by every P V issued so far
      commit(br.kv_empty(vs));
      if (more) {
        // probe what the next step needs, then issue S1 for it
        const bool raw_v =
            mbar_test_wait(br.kv_full((kv_it + 2) % G::NS), ((kv_it + 2) / G::NS) & 1u);
        const bool raw_k =
            idx + 2 < n
                ? mbar_test_wait(br.kv_full((kv_it + 3) % G::NS), ((kv_it + 3) / G::NS) & 1u)
                : true;
        const bool raw_p0 = mbar_test_wait(br.p_half(0), pf_phase0);
        if (x.valid1) {
          issue_qk(1, ks);
          commit(br.s_full(1));
        }
        rdy_v = __all_sync(0xffffffffu, raw_v);
        rdy_k = __all_sync(0xffffffffu, raw_k);
        rdy_p0 = __all_sync(0xffffffffu, raw_p0);
        commit(br.kv_empty(ks));
        if (idx + 1 == n - 1) commit(br.q_empty);
      }
      kv_it += more ? 2u : 1u;
    }
    ++units0;
    if (x.valid1) ++units1;
  }
  return;
drain:
  commit(br.drain);
  if (leader) drain_wait(br.drain, 0u, 200000000ull);
  __syncwarp();
}

}  // namespace ra
