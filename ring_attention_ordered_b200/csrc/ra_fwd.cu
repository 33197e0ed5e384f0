// Forward ring-ordered blockwise attention for sm_100a.
//
// What it computes ("Ring Attention 环注意力", slowleelab ai-terms-fun):
//   * the sequence is cut into n_ring equal blocks (L4 §4.2 setup);
//   * the query block of host i visits K/V blocks j = (i - t) mod n_ring,
//     t = 0..n_ring-1 (L3 definition, L4 §4.2);
//   * each visit is exact blockwise attention folded into a running
//     online-softmax accumulator (L4 §4.3; the recurrence of the
//     FlashAttention article, 核心原理), with one normalisation at the end;
//   * causal: visits j > i skipped, j == i diagonal-masked, j < i unmasked
//     (L4 §4.5, limitation 2);
//   * fp32 statistics and accumulators (L5 §5.2, pitfall 9);
//   * grouped-query heads share K/V tiles (lnwmold page §2.2).
//
// How (B200 design):
//   * persistent CTAs, one per SM, each owning a static, snake-ordered share
//     of work units sorted longest-first (the causal load balance of L4 §4.5,
//     limitation 3); a unit is two 128-row query tiles that see the same K/V
//     stream -- two heads of one GQA group at the same rows, or two adjacent
//     tiles of one head inside one ring block;
//   * warp 8 loads Q/K/V tiles with TMA (128-byte swizzle) into a K/V ring of
//     shared-memory stages;
//   * warp 9 (one thread) issues tcgen05.mma: S_w = Q_w K^T into TMEM, then
//     O_w += P_w V with P_w read from TMEM;
//   * warps 0-3 and 4-7 each own one query tile (one TMEM lane = one row):
//     they read S, apply the mask, keep the running max/sum in fp32, write P
//     as bf16 back over S, rescale O in TMEM only when the running max grew by
//     more than 2^8 (the final division cancels a stale max exactly), and run
//     the epilogue O / l, lse = m + ln l.  The two tiles ping-pong, so one
//     tile's softmax runs under the other tile's MMAs (the overlap the
//     FlashAttention article describes for FlashAttention-3);
//   * every mbarrier wait is bounded by %globaltimer; a wait that runs out
//     records RA_ERR_TIMEOUT in a device status word, the CTA drains its
//     in-flight copies and MMAs, frees its TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>

#include "ptx_sm100.cuh"
#include "ra_internal.h"
#include "ring_attn.h"

namespace ra {

constexpr int BM = 128;             // query rows per tile
constexpr int BN = 128;             // keys per K/V tile
constexpr int BOX_COLS = 64;        // TMA box width (64 bf16 = one 128-byte swizzle row)
constexpr int BOX_BYTES = 128 * 128;
constexpr int NUM_THREADS = 384;   // three warpgroups
constexpr int WARP_LOAD = 8;
constexpr int WARP_MMA = 9;
// Register split (setmaxnreg): the kernel launches with LAUNCH_REGS per
// thread; the control warpgroup (warps 8-11) gives registers back and the two
// softmax warpgroups take them.  The shares must add up to at most the launch
// total, which the host checks before the first launch.
constexpr int LAUNCH_REGS = 168;
constexpr int SOFTMAX_REGS = 216;
constexpr int CONTROL_REGS = 72;
static_assert(2 * 128 * SOFTMAX_REGS + 128 * CONTROL_REGS <= NUM_THREADS * LAUNCH_REGS,
              "register split exceeds the launch allocation");
constexpr float RESCALE_LOG2 = 8.0f;
constexpr float LN2 = 0.69314718055994530942f;

// Device status word: 0 = ok, otherwise (code << 32) | where.
__device__ unsigned long long g_ra_status = 0ull;

enum WaitSite : uint32_t {
  SITE_Q_FULL = 1, SITE_Q_EMPTY, SITE_KV_FULL, SITE_KV_EMPTY, SITE_S_FULL,
  SITE_P_FULL, SITE_O_DONE, SITE_O_FREE
};

template <int D>
struct Cfg {
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int NS = (D == 128) ? 4 : 8;   // K/V stages
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = 2 * Q_BYTES;
  static constexpr int OFF_BAR = OFF_KV + NS * KV_BYTES;
  // barriers: q_full, q_empty, kv_full[NS], kv_empty[NS], s_full[2],
  // p_full[2], o_done[2], o_free[2], drain; then tmem holder + abort flag
  static constexpr int NUM_BARS = 2 + 2 * NS + 8 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct Unit {
  int b, kvh, blk;
  int h[2];
  int qt[2];       // tile index inside ring block blk
  int valid1;
  int qt_last;
  int n_kv;        // K/V tiles visited, in ring order
};

__device__ __forceinline__ Unit decode_unit(const FwdParams& p, long long u) {
  Unit x;
  const int tpb = p.tiles_per_blk;
  if (p.pair_heads) {
    const long long per_tile = static_cast<long long>(p.B) * p.Hkv * p.head_slots;
    const long long r = u / per_tile;
    long long rem = u % per_tile;
    const int gt = p.n_ring * tpb - 1 - static_cast<int>(r);   // longest first
    x.blk = gt / tpb;
    const int local = gt % tpb;
    const int slot = static_cast<int>(rem % p.head_slots);
    rem /= p.head_slots;
    x.kvh = static_cast<int>(rem % p.Hkv);
    x.b = static_cast<int>(rem / p.Hkv);
    x.h[0] = x.kvh * p.group + 2 * slot;
    x.h[1] = x.h[0] + 1;
    x.valid1 = (2 * slot + 1) < p.group;
    x.qt[0] = x.qt[1] = local;
  } else {
    const long long per_pair = static_cast<long long>(p.B) * p.Hq;
    const long long r = u / per_pair;
    const int bh = static_cast<int>(u % per_pair);
    x.b = bh / p.Hq;
    x.h[0] = x.h[1] = bh % p.Hq;
    x.kvh = x.h[0] / p.group;
    const int ppb = p.pairs_per_blk;
    x.blk = p.n_ring - 1 - static_cast<int>(r / ppb);
    const int pr = ppb - 1 - static_cast<int>(r % ppb);
    x.qt[0] = 2 * pr;
    x.qt[1] = 2 * pr + 1;
    x.valid1 = x.qt[1] < tpb;
  }
  x.qt_last = x.valid1 ? max(x.qt[0], x.qt[1]) : x.qt[0];
  x.n_kv = p.causal ? (x.blk * tpb + x.qt_last + 1) : (p.n_ring * tpb);
  return x;
}

// idx-th K/V tile of a unit: its ring block j (returned in jb) and its tile
// index inside that block.  The unit's own block comes first (step t = 0),
// then blocks (i - t) mod n_ring for t = 1, 2, ...; inside a block the tiles
// run in ascending order, and under causal masking the own block stops at the
// unit's last query tile.
__device__ __forceinline__ int kv_tile_at(const FwdParams& p, const Unit& x, int idx, int& jb) {
  const int tpb = p.tiles_per_blk;
  const int ndiag = p.causal ? (x.qt_last + 1) : tpb;
  if (idx < ndiag) {
    jb = x.blk;
    return idx;
  }
  const int r = idx - ndiag;
  const int step = 1 + r / tpb;
  jb = (x.blk - step + p.n_ring) % p.n_ring;
  return r % tpb;
}

// Static persistent schedule: in round k, CTA c takes unit k*G + c (k even)
// or k*G + G-1-c (k odd).  Units are sorted longest first, so the snake keeps
// the per-CTA totals within about one unit of each other.
__device__ __forceinline__ long long unit_for_round(long long k, int G, int c) {
  return k * G + ((k & 1) ? (G - 1 - c) : c);
}

struct Ctl {
  volatile uint32_t* abort;
  unsigned long long limit_ns;
};

__device__ __noinline__ void record_timeout(const Ctl& cx, uint32_t site) {
  *cx.abort = 1u;
  const unsigned long long code =
      (static_cast<unsigned long long>(RA_ERR_TIMEOUT) << 32) | (site << 16) | (blockIdx.x & 0xFFFF);
  atomicCAS(&g_ra_status, 0ull, code);
}

// Bounded wait on an mbarrier phase.  Returns false if the kernel is aborting
// (this wait ran out, or another role's did).
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, const Ctl& cx,
                                         uint32_t site) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  uint32_t spins = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*cx.abort) return false;
    if ((++spins & 31u) == 0u && globaltimer_ns() - t0 > cx.limit_ns) {
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

struct Bars {
  uint32_t q_full, q_empty, kv_full0, kv_empty0, s_full0, p_full0, o_done0, o_free0, drain;
  __device__ __forceinline__ uint32_t kv_full(int s) const { return kv_full0 + 8u * s; }
  __device__ __forceinline__ uint32_t kv_empty(int s) const { return kv_empty0 + 8u * s; }
  __device__ __forceinline__ uint32_t s_full(int w) const { return s_full0 + 8u * w; }
  __device__ __forceinline__ uint32_t p_full(int w) const { return p_full0 + 8u * w; }
  __device__ __forceinline__ uint32_t o_done(int w) const { return o_done0 + 8u * w; }
  __device__ __forceinline__ uint32_t o_free(int w) const { return o_free0 + 8u * w; }
};

// ------------------------------------------------------------------ loader
template <int D>
__device__ void loader_role(const FwdParams& p, const Bars& br, uint32_t smem_base, const Ctl& cx) {
  using C = Cfg<D>;
  constexpr int NBOX = D / BOX_COLS;
  const int G = gridDim.x, c = blockIdx.x;
  uint32_t kv_it = 0, q_uses = 0;
  bool q_pending = false;
  for (long long k = 0;; ++k) {
    const long long u = unit_for_round(k, G, c);
    if (u >= p.total_units) break;
    const Unit x = decode_unit(p, u);
    if (q_uses > 0 && !wait_bar(br.q_empty, (q_uses - 1) & 1u, cx, SITE_Q_EMPTY)) goto drain;
    if ((p.debug_flags & 1u) && q_uses == 0) {
      // fault injection: the first query tiles are never requested
    } else {
      const int nq = x.valid1 ? 2 : 1;
      mbar_arrive_expect_tx(br.q_full, nq * C::Q_BYTES);
      for (int w = 0; w < nq; ++w) {
        const int row = x.b * p.L + x.blk * p.blk_len + x.qt[w] * BM;
        for (int bx = 0; bx < NBOX; ++bx)
          tma_load_3d(smem_base + C::OFF_Q + w * C::Q_BYTES + bx * BOX_BYTES, &p.tm_q, br.q_full,
                      bx * BOX_COLS, x.h[w], row);
      }
      q_pending = true;
    }
    ++q_uses;
    for (int idx = 0; idx < x.n_kv; ++idx) {
      int jb;
      const int kl = kv_tile_at(p, x, idx, jb);
      const int row = x.b * p.L + jb * p.blk_len + kl * BN;
      for (int kv = 0; kv < 2; ++kv) {
        const int s = kv_it % C::NS;
        const uint32_t ph = (kv_it / C::NS) & 1u;
        if (!wait_bar(br.kv_empty(s), ph ^ 1u, cx, SITE_KV_EMPTY)) goto drain;
        mbar_arrive_expect_tx(br.kv_full(s), C::KV_BYTES);
        const CUtensorMap* map = kv ? &p.tm_v : &p.tm_k;
        for (int bx = 0; bx < NBOX; ++bx)
          tma_load_3d(smem_base + C::OFF_KV + s * C::KV_BYTES + bx * BOX_BYTES, map, br.kv_full(s),
                      bx * BOX_COLS, x.kvh, row);
        ++kv_it;
      }
    }
  }
  return;
drain:
  // Let the copies already issued land before the CTA's shared memory goes.
  {
    const uint32_t n = kv_it < static_cast<uint32_t>(C::NS) ? kv_it : C::NS;
    for (uint32_t i = 0; i < n; ++i) {
      const uint32_t it = kv_it - 1 - i;
      drain_wait(br.kv_full(it % C::NS), (it / C::NS) & 1u, 200000000ull);
    }
    if (q_pending) drain_wait(br.q_full, (q_uses - 1) & 1u, 200000000ull);
  }
}

// ------------------------------------------------------------------ MMA
template <int D>
__device__ void mma_role(const FwdParams& p, const Bars& br, uint32_t smem_base, uint32_t tmem,
                         const Ctl& cx) {
  using C = Cfg<D>;
  constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, false);
  constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, true);
  const int G = gridDim.x, c = blockIdx.x;
  uint32_t kv_it = 0, q_uses = 0;
  uint32_t pf_phase[2] = {0u, 0u};
  uint32_t units_w[2] = {0u, 0u};

  // Descriptor start addresses are in 16-byte units in the low 14 bits; all
  // shared-memory offsets here stay below 2^18 bytes, so adding (offset >> 4)
  // to a base descriptor never carries out of that field.
  const uint64_t dq0 = smem_desc_sw128(smem_base + C::OFF_Q, 16, 1024);
  const uint64_t dkv0 = smem_desc_sw128(smem_base + C::OFF_KV, 16, 1024);
  const uint64_t dv0 = smem_desc_sw128(smem_base + C::OFF_KV, BOX_BYTES, 1024);
  auto issue_qk = [&](int w, int stage) {
    const uint64_t dq = dq0 + static_cast<uint32_t>((w * C::Q_BYTES) >> 4);
    const uint64_t dk = dkv0 + static_cast<uint32_t>((stage * C::KV_BYTES) >> 4);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t off = ((kk / 4) * BOX_BYTES + (kk % 4) * 32) >> 4;
      mma_ss(tmem + w * 128, dq + off, dk + off, IDESC_QK, kk > 0 ? 1u : 0u);
    }
  };
  auto issue_pv = [&](int w, int stage, bool acc) {
    const uint64_t dv = dv0 + static_cast<uint32_t>((stage * C::KV_BYTES) >> 4);
#pragma unroll
    for (int kk = 0; kk < BN / 16; ++kk) {
      mma_ts(tmem + 256 + w * 128, tmem + w * 128 + kk * 8, dv + static_cast<uint32_t>(kk * 128),
             IDESC_PV, (acc || kk > 0) ? 1u : 0u);
    }
  };

  for (long long k = 0;; ++k) {
    const long long u = unit_for_round(k, G, c);
    if (u >= p.total_units) break;
    const Unit x = decode_unit(p, u);
    const int n = x.n_kv;
    if (!wait_bar(br.q_full, q_uses & 1u, cx, SITE_Q_FULL)) goto drain;
    tc_fence_after();
    ++q_uses;
    {
      const int ks = kv_it % C::NS;
      if (!wait_bar(br.kv_full(ks), (kv_it / C::NS) & 1u, cx, SITE_KV_FULL)) goto drain;
      tc_fence_after();
      issue_qk(0, ks);
      tc_commit(br.s_full(0));
      if (x.valid1) {
        issue_qk(1, ks);
        tc_commit(br.s_full(1));
      }
      tc_commit(br.kv_empty(ks));
      ++kv_it;
      if (n == 1) tc_commit(br.q_empty);
    }
    for (int idx = 0; idx < n; ++idx) {
      const bool more = idx + 1 < n;
      const int vs = kv_it % C::NS;
      const int ks = (kv_it + 1) % C::NS;
      if (!wait_bar(br.kv_full(vs), (kv_it / C::NS) & 1u, cx, SITE_KV_FULL)) goto drain;
      tc_fence_after();
      for (int w = 0; w < 2; ++w) {
        if (w == 1 && !x.valid1) break;
        if (!wait_bar(br.p_full(w), pf_phase[w], cx, SITE_P_FULL)) goto drain;
        pf_phase[w] ^= 1u;
        tc_fence_after();
        if (idx == 0 && units_w[w] > 0) {
          if (!wait_bar(br.o_free(w), (units_w[w] - 1) & 1u, cx, SITE_O_FREE)) goto drain;
          tc_fence_after();
        }
        issue_pv(w, vs, idx > 0);
        if (!more) tc_commit(br.o_done(w));
        if (more) {
          if (w == 0) {
            if (!wait_bar(br.kv_full(ks), ((kv_it + 1) / C::NS) & 1u, cx, SITE_KV_FULL)) goto drain;
            tc_fence_after();
          }
          issue_qk(w, ks);
          tc_commit(br.s_full(w));
        }
      }
      tc_commit(br.kv_empty(vs));
      if (more) {
        tc_commit(br.kv_empty(ks));
        if (idx + 1 == n - 1) tc_commit(br.q_empty);
      }
      kv_it += more ? 2u : 1u;
    }
    ++units_w[0];
    if (x.valid1) ++units_w[1];
  }
  return;
drain:
  tc_commit(br.drain);
  drain_wait(br.drain, 0u, 200000000ull);
}

// ------------------------------------------------------------------ softmax
template <int D>
__device__ void softmax_role(const FwdParams& p, const Bars& br, uint32_t tmem, int w,
                             const Ctl& cx) {
  const int t = threadIdx.x - w * 128;            // row inside the query tile
  const int quarter = (threadIdx.x >> 5) & 3;     // TMEM lane quarter of this warp
  const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t tS = tmem + lane_off + w * 128;  // S (fp32) and P (bf16 pairs, first 64 cols)
  const uint32_t tO = tmem + lane_off + 256 + w * 128;
  const float c2 = p.scale_log2;
  const int G = gridDim.x, cta = blockIdx.x;
  uint32_t s_phase = 0u, units_w = 0u;

  for (long long k = 0;; ++k) {
    const long long u = unit_for_round(k, G, cta);
    if (u >= p.total_units) break;
    const Unit x = decode_unit(p, u);
    if (w == 1 && !x.valid1) continue;
    const int qt = x.qt[w];
    const int h = x.h[w];
    const int qrow = qt * BM + t;                  // row inside the ring block
    float m = -INFINITY, l = 0.f;

    for (int idx = 0; idx < x.n_kv; ++idx) {
      int jb;
      const int kl = kv_tile_at(p, x, idx, jb);
      bool ok = wait_bar(br.s_full(w), s_phase, cx, SITE_S_FULL);
      if (!__all_sync(0xffffffffu, ok)) return;
      s_phase ^= 1u;
      tc_fence_after();

      uint32_t sr[128];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t (&chunk)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[cc * 32]);
        tmem_ld32(tS + cc * 32, chunk);
      }
      tmem_wait_ld();

      // keys allowed for this row: columns 0..lim of the tile
      int lim = min(BN, p.blk_len - kl * BN) - 1;
      if (p.causal && jb == x.blk) lim = min(lim, qrow - kl * BN);
      const bool masked = lim < BN - 1;

      float mx[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx[i] = -INFINITY;
      if (!masked) {
#pragma unroll
        for (int j = 0; j < 128; ++j) mx[j & 7] = fmaxf(mx[j & 7], __uint_as_float(sr[j]));
      } else {
#pragma unroll
        for (int j = 0; j < 128; ++j) {
          if (j > lim) sr[j] = __float_as_uint(-INFINITY);
          mx[j & 7] = fmaxf(mx[j & 7], __uint_as_float(sr[j]));
        }
      }
      float rmax = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                         fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      const float m_tile = (rmax == -INFINITY) ? -INFINITY : rmax * c2;
      const bool need = m_tile > m + RESCALE_LOG2;
      const float m_new = need ? m_tile : m;
      const float alpha = (m_new == m) ? 1.f : ex2_approx(m - m_new);
      if (idx > 0 && __any_sync(0xffffffffu, need)) {
        // O already holds every earlier P V of this tile: the commit that
        // signalled S for this step fires only after them.
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + cc * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
          tmem_st32(tO + cc * 32, o);
        }
        tmem_wait_st();
      }
      m = m_new;
      l *= alpha;

      const float neg_m = -m;
      float rs[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) rs[i] = 0.f;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int c0 = 64 * half + 2 * j;
          float p0 = ex2_approx(fmaf(__uint_as_float(sr[c0]), c2, neg_m));
          float p1 = ex2_approx(fmaf(__uint_as_float(sr[c0 + 1]), c2, neg_m));
          if (masked) {
            p0 = (c0 > lim) ? 0.f : p0;
            p1 = (c0 + 1 > lim) ? 0.f : p1;
          }
          rs[j & 7] += p0 + p1;
          pk[j] = pack_bf16x2(p0, p1);
        }
        tmem_st32(tS + 32 * half, pk);
      }
      l += ((rs[0] + rs[1]) + (rs[2] + rs[3])) + ((rs[4] + rs[5]) + (rs[6] + rs[7]));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(br.p_full(w));
    }

    // epilogue: wait for the last P V, then O / l and lse = m + ln l
    {
      bool ok = wait_bar(br.o_done(w), units_w & 1u, cx, SITE_O_DONE);
      if (!__all_sync(0xffffffffu, ok)) return;
      tc_fence_after();
      const bool row_ok = qrow < p.blk_len;
      const long long pos = static_cast<long long>(x.blk) * p.blk_len + qrow;
      const float inv_l = 1.f / l;
      __nv_bfloat16* dst = p.out + ((static_cast<long long>(x.b) * p.L + pos) * p.Hq + h) * D;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tmem_ld32(tO + cc * 32, o);
        tmem_wait_ld();
        uint32_t pkd[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          pkd[j] = pack_bf16x2(__uint_as_float(o[2 * j]) * inv_l, __uint_as_float(o[2 * j + 1]) * inv_l);
        if (row_ok) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + cc * 32);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            d4[j] = make_uint4(pkd[4 * j], pkd[4 * j + 1], pkd[4 * j + 2], pkd[4 * j + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(br.o_free(w));
      if (row_ok)
        p.lse[(static_cast<long long>(x.b) * p.Hq + h) * p.L + pos] = (m + log2f(l)) * LN2;
      ++units_w;
    }
  }
}

// ------------------------------------------------------------------ kernel
template <int D>
__global__ void __launch_bounds__(NUM_THREADS, 1) ra_fwd_kernel(const __grid_constant__ FwdParams p) {
  using C = Cfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);

  Bars br;
  br.q_full = base + C::OFF_BAR;
  br.q_empty = br.q_full + 8;
  br.kv_full0 = br.q_empty + 8;
  br.kv_empty0 = br.kv_full0 + 8 * C::NS;
  br.s_full0 = br.kv_empty0 + 8 * C::NS;
  br.p_full0 = br.s_full0 + 16;
  br.o_done0 = br.p_full0 + 16;
  br.o_free0 = br.o_done0 + 16;
  br.drain = br.o_free0 + 16;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(base_ptr + C::OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(base_ptr + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(br.q_full, 1);
    mbar_init(br.q_empty, 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(br.kv_full(s), 1);
      mbar_init(br.kv_empty(s), 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(br.s_full(w), 1);
      mbar_init(br.p_full(w), 128);
      mbar_init(br.o_done(w), 1);
      mbar_init(br.o_free(w), 128);
    }
    mbar_init(br.drain, 1);
    *abort_flag = 0u;
    fence_mbarrier_init();
  }
  if (warp == WARP_LOAD && lane == 0) {
    prefetch_tensormap(&p.tm_q);
    prefetch_tensormap(&p.tm_k);
    prefetch_tensormap(&p.tm_v);
  }
  if (warp == WARP_MMA) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const Ctl cx{abort_flag, p.wait_limit_ns};

  if (warp < 8) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" :: "n"(SOFTMAX_REGS));
    softmax_role<D>(p, br, tmem, warp >> 2, cx);
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" :: "n"(CONTROL_REGS));
    if (warp == WARP_LOAD) {
      if (lane == 0) loader_role<D>(p, br, base, cx);
    } else if (warp == WARP_MMA) {
      if (lane == 0) mma_role<D>(p, br, base, tmem, cx);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ host
template <int D>
static cudaError_t launch_fwd_d(const FwdParams& prm, int grid, cudaStream_t stream) {
  using C = Cfg<D>;
  static int configured_dev[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured_dev[dev]) {
    // The setmaxnreg split is only safe if the kernel really launches with
    // LAUNCH_REGS registers per thread; refuse to launch otherwise.
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, ra_fwd_kernel<D>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != LAUNCH_REGS) return cudaErrorInvalidKernelImage;
    e = cudaFuncSetAttribute(ra_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    configured_dev[dev] = 1;
  }
  ra_fwd_kernel<D><<<grid, NUM_THREADS, C::SMEM_BYTES, stream>>>(prm);
  return cudaGetLastError();
}

cudaError_t launch_fwd(const FwdParams& prm, int d, int grid, cudaStream_t stream) {
  if (d == 128) return launch_fwd_d<128>(prm, grid, stream);
  return launch_fwd_d<64>(prm, grid, stream);
}

cudaError_t read_and_clear_status(unsigned long long* out) {
  unsigned long long v = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_ra_status, sizeof(v));
  if (e != cudaSuccess) return e;
  if (v != 0) {
    e = cudaMemcpyToSymbol(g_ra_status, &zero, sizeof(zero));
    if (e != cudaSuccess) return e;
  }
  *out = v;
  return cudaSuccess;
}

}  // namespace ra
