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
//   * persistent CTAs, one per SM, taking work units from a queue shared by
//     the launch (an atomic counter over units sorted longest first, the
//     causal load balance of L4 §4.5, limitation 3), so that all CTAs stay
//     within about one unit of each other and the K/V heads they read stay
//     few; a unit is two 128-row query tiles that see the same K/V stream --
//     two heads of one GQA group at the same rows, or two adjacent tiles of
//     one head inside one ring block;
//   * warp 8 loads Q/K/V tiles with TMA (128-byte swizzle) into a K/V ring of
//     shared-memory stages;
//   * warp 9 (one thread) issues tcgen05.mma: S_w = Q_w K^T into TMEM, then
//     O_w += P_w V with P_w read from TMEM;
//   * warps 0-3 and 4-7 each own one query tile (one TMEM lane = one row):
//     they read S, apply the mask, keep the running max/sum in fp32, write P
//     as bf16 back over S, rescale O in TMEM whenever the running max grows
//     by more than a factor 2 (so a dominant key has P = 1 exactly), and run
//     the epilogue O / l, lse = m + ln l.  The two tiles ping-pong, so one
//     tile's softmax runs under the other tile's MMAs (the overlap the
//     FlashAttention article describes for FlashAttention-3);
//   * every mbarrier wait is bounded by %globaltimer; a wait that runs out
//     records RA_ERR_TIMEOUT in a device status word, the CTA drains its
//     in-flight copies and MMAs, frees its TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstdio>

#include "ptx_sm100.cuh"
#include "ra_fwd_roles.cuh"
#include "ra_internal.h"
#include "ra_merge_math.cuh"
#include "ra_schedule.cuh"
#include "ra_sync.cuh"
#include "ring_attn.h"

namespace ra {

constexpr int BM = FWD_BM;          // query rows per tile
constexpr int BN = FWD_BN;          // keys per K/V tile
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
constexpr int SOFTMAX_REGS = 224;
constexpr int CONTROL_REGS = 56;
static_assert(2 * 128 * SOFTMAX_REGS + 128 * CONTROL_REGS <= NUM_THREADS * LAUNCH_REGS,
              "register split exceeds the launch allocation");
// The reference maximum follows the row's running maximum closely: O and l
// are rescaled whenever a tile raises it by more than a factor 2 (1 in log2
// units).  A key that dominates its row stands that far above the earlier
// maximum, so it sets the reference and gets P = 2^0 = 1, exact in bf16: its
// weight carries no bf16 rounding into O.  (A reference moved only past 2^8
// leaves such a key's P in (1, 256], and that P's bf16 rounding, up to 2^-9
// relative, shows in O; following every rise of the maximum costs O
// rescales in many more steps for the same accuracy.)
constexpr float RESCALE_LOG2 = 1.0f;
constexpr float LN2 = 0.69314718055994530942f;

// Device status word: 0 = ok, otherwise (code << 32) | where.
__device__ unsigned long long g_ra_status = 0ull;

// Work-queue counters of the forward launches (see next_ticket_counter).
__device__ unsigned int g_ra_tickets[kTicketSlots];

// Shared-memory layout (D = head dim): Q0, Q1, NS K/V stages, barriers, the
// TMEM holder and abort flag, the unit queue.
template <int D>
struct Cfg {
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int NS = (D == 128) ? 4 : 8;   // K/V stages
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = 2 * Q_BYTES;
  static constexpr int OFF_BAR = OFF_KV + NS * KV_BYTES;
  static constexpr int OFF_MISC = OFF_BAR + fwd_num_bars(NS) * 8;
  static constexpr int OFF_UNITS = OFF_MISC + 16;
  static constexpr int SMEM_BYTES = OFF_UNITS + UQ * 4 + 1024;  // + alignment slack
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// ------------------------------------------------------------------ MMA
template <int KK>
struct QkStep {
  static constexpr uint32_t OFF = ((KK / 4) * BOX_BYTES + (KK % 4) * 32) >> 4;
};

// S = Q K^T over the head dimension: D/16 MMAs of K = 16, each issued by
// the elected lane.
template <int D>
__device__ __forceinline__ void mma_qk_steps(uint32_t d, uint32_t a, uint32_t b, uint32_t hi,
                                             uint32_t idesc) {
  if (elect_one()) mma_ss<QkStep<0>::OFF, QkStep<0>::OFF>(d, a, hi, b, hi, idesc, 0u);
  if (elect_one()) mma_ss<QkStep<1>::OFF, QkStep<1>::OFF>(d, a, hi, b, hi, idesc, 1u);
  if (elect_one()) mma_ss<QkStep<2>::OFF, QkStep<2>::OFF>(d, a, hi, b, hi, idesc, 1u);
  if (elect_one()) mma_ss<QkStep<3>::OFF, QkStep<3>::OFF>(d, a, hi, b, hi, idesc, 1u);
  if constexpr (D == 128) {
    if (elect_one()) mma_ss<QkStep<4>::OFF, QkStep<4>::OFF>(d, a, hi, b, hi, idesc, 1u);
    if (elect_one()) mma_ss<QkStep<5>::OFF, QkStep<5>::OFF>(d, a, hi, b, hi, idesc, 1u);
    if (elect_one()) mma_ss<QkStep<6>::OFF, QkStep<6>::OFF>(d, a, hi, b, hi, idesc, 1u);
    if (elect_one()) mma_ss<QkStep<7>::OFF, QkStep<7>::OFF>(d, a, hi, b, hi, idesc, 1u);
  }
}

// O (+)= P V over one half of the 128 keys (HALF 0: keys 0-63, 1: keys
// 64-127): 4 MMAs of K = 16; P's 16 keys are 8 TMEM columns of bf16 pairs,
// V's 16 keys are 16 rows of 128 bytes (2048 bytes).  `acc` applies to the
// first MMA of the first half only.
template <int HALF>
__device__ __forceinline__ void mma_pv_half(uint32_t d, uint32_t p_tmem, uint32_t b, uint32_t hi,
                                            uint32_t idesc, uint32_t acc) {
  constexpr uint32_t C0 = 32 * HALF, B0 = 512 * HALF;
  if (elect_one()) mma_ts<C0 + 0, B0 + 0>(d, p_tmem, b, hi, idesc, HALF ? 1u : acc);
  if (elect_one()) mma_ts<C0 + 8, B0 + 128>(d, p_tmem, b, hi, idesc, 1u);
  if (elect_one()) mma_ts<C0 + 16, B0 + 256>(d, p_tmem, b, hi, idesc, 1u);
  if (elect_one()) mma_ts<C0 + 24, B0 + 384>(d, p_tmem, b, hi, idesc, 1u);
}

// Geometry of the bf16 kernel for the shared loader and MMA roles: a tile
// row of D bf16 values is D / 64 TMA boxes of 64 columns (one 128-byte
// swizzle row each), BOX_BYTES apart; tcgen05.mma kind::f16 with K = 16.
template <int D>
struct Bf16Geom {
  using C = Cfg<D>;
  static constexpr int Q_BYTES = C::Q_BYTES;
  static constexpr int KV_BYTES = C::KV_BYTES;
  static constexpr int NS = C::NS;
  static constexpr int OFF_Q = C::OFF_Q;
  static constexpr int OFF_KV = C::OFF_KV;
  static constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, true);

  static __device__ __forceinline__ void load_tile(uint32_t dst, const CUtensorMap* map,
                                                   uint32_t bar, int h, int row) {
#pragma unroll
    for (int bx = 0; bx < D / BOX_COLS; ++bx)
      tma_load_3d(dst + bx * BOX_BYTES, map, bar, bx * BOX_COLS, h, row);
  }
  static __device__ __forceinline__ void load_q(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                                int h, int row) {
    load_tile(dst, map, bar, h, row);
  }
  static __device__ __forceinline__ void load_kv(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t bar, int h, int row) {
    load_tile(dst, map, bar, h, row);
  }

  // Shared-memory descriptors as (low, high) words.  The start address sits
  // in the low 14 bits in 16-byte units; every offset used here keeps the
  // address below 2^18 bytes, so adding (offset >> 4) to the low word never
  // carries out of that field.  The high words are fixed by the layout.
  uint32_t q_lo, k_lo, v_lo, k_hi, v_hi;
  __device__ explicit Bf16Geom(uint32_t smem_base) {
    const uint64_t dq0 = smem_desc_sw128(smem_base + OFF_Q, 16, 1024);
    const uint64_t dkv0 = smem_desc_sw128(smem_base + OFF_KV, 16, 1024);
    const uint64_t dv0 = smem_desc_sw128(smem_base + OFF_KV, BOX_BYTES, 1024);
    q_lo = static_cast<uint32_t>(dq0);
    k_lo = static_cast<uint32_t>(dkv0);
    v_lo = static_cast<uint32_t>(dv0);
    k_hi = static_cast<uint32_t>(dkv0 >> 32);
    v_hi = static_cast<uint32_t>(dv0 >> 32);
  }
  // S_w = Q_w K^T into TMEM at d: k-steps of 16 elements, 32 bytes apart
  // inside a 64-column swizzle box, the next box BOX_BYTES further on.
  __device__ __forceinline__ void issue_qk(uint32_t d, int w, int stage) const {
    mma_qk_steps<D>(d, q_lo + ((w * Q_BYTES) >> 4), k_lo + ((stage * KV_BYTES) >> 4), k_hi,
                    IDESC_QK);
  }
  // O_w (+)= P_w V over keys 64 HALF .. 64 HALF + 63.
  template <int HALF>
  __device__ __forceinline__ void issue_pv_half(uint32_t d, uint32_t p_tmem, int stage,
                                                uint32_t acc) const {
    mma_pv_half<HALF>(d, p_tmem, v_lo + ((stage * KV_BYTES) >> 4), v_hi, IDESC_PV, acc);
  }
};

// ------------------------------------------------------------------ softmax
// One score row (128 columns held in sr): P = 2^(s * c2 - m) written as bf16
// pairs to TMEM columns [0, 64) at tS, returns the row sum of the fp32 P.
// Arrives on p_half_bar once the first 64 keys of P are stored.
// MASKED: columns > lim are excluded (set to zero exactly).  Issues
// warp-collective tcgen05.st: every lane of the warp must call the same
// instantiation at the same time.
template <bool MASKED>
__device__ __forceinline__ float exp_row_store(uint32_t (&sr)[128], float c2, float m, int lim,
                                               uint32_t tS, uint32_t p_half_bar) {
  const uint64_t c2x2 = f2_pack(c2, c2);
  const uint64_t nm2 = f2_pack(-m, -m);
  uint64_t acc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i] = f2_pack(0.f, 0.f);
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    uint32_t pk[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int col = 64 * half + 2 * j;
      const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(sr[col]), __uint_as_float(sr[col + 1])),
                                 c2x2, nm2);
      float p0, p1;
      f2_unpack(x2, p0, p1);
      p0 = ex2_approx(p0);
      p1 = ex2_approx(p1);
      if (MASKED) {
        p0 = (col > lim) ? 0.f : p0;
        p1 = (col + 1 > lim) ? 0.f : p1;
      }
      acc[j & 3] = f2_add(acc[j & 3], f2_pack(p0, p1));
      pk[j] = pack_bf16x2(p0, p1);
    }
    tmem_st32(tS + 32 * half, pk);
    if (half == 0) {
      // the first 64 keys of P are in TMEM: let the MMA start on them
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_half_bar);
    }
  }
  const uint64_t s01 = f2_add(acc[0], acc[1]);
  const uint64_t s23 = f2_add(acc[2], acc[3]);
  float a, b;
  f2_unpack(f2_add(s01, s23), a, b);
  return a + b;
}

// Epilogue of a per-visit launch: this visit's normalised rows O / l (fp32)
// are folded into the running accumulator o_acc / lse with the row merge of
// the merge kernel (bitwise the same as writing them and merging), or
// overwrite it on the first visit; `out` optionally gets the bf16 rounding.
// The accumulator row was prefetched into L2 during the unit's last K/V step.
template <int D>
__device__ __forceinline__ void visit_epilogue(const FwdParams& p, uint32_t tO, bool row_ok, int b,
                                               long long pos, int h, float inv_l, float lse_t) {
  const long long row = (static_cast<long long>(b) * p.L + pos) * p.Hq + h;
  float* lse_dst = p.lse + (static_cast<long long>(b) * p.Hq + h) * p.L + pos;
  float4* acc = reinterpret_cast<float4*>(p.o_acc + row * D);
  uint4* out4 = reinterpret_cast<uint4*>(p.out + row * D);
  MergeW mw;
  if (p.visit_fold && row_ok) mw = merge_weights(*lse_dst, lse_t);
#pragma unroll
  for (int cc = 0; cc < D / 32; ++cc) {
    uint32_t o[32];
    tmem_ld32(tO + cc * 32, o);
    tmem_wait_ld();
    float r[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) r[j] = __uint_as_float(o[j]) * inv_l;
    if (row_ok) {
      if (p.visit_fold) {
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          const float4 a = acc[cc * 8 + c4];
          r[4 * c4 + 0] = merge_one(mw, a.x, r[4 * c4 + 0]);
          r[4 * c4 + 1] = merge_one(mw, a.y, r[4 * c4 + 1]);
          r[4 * c4 + 2] = merge_one(mw, a.z, r[4 * c4 + 2]);
          r[4 * c4 + 3] = merge_one(mw, a.w, r[4 * c4 + 3]);
        }
      }
#pragma unroll
      for (int c4 = 0; c4 < 8; ++c4)
        acc[cc * 8 + c4] = make_float4(r[4 * c4], r[4 * c4 + 1], r[4 * c4 + 2], r[4 * c4 + 3]);
      if (p.out != nullptr) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          out4[cc * 4 + j] =
              make_uint4(pack_bf16x2(r[8 * j], r[8 * j + 1]), pack_bf16x2(r[8 * j + 2], r[8 * j + 3]),
                         pack_bf16x2(r[8 * j + 4], r[8 * j + 5]),
                         pack_bf16x2(r[8 * j + 6], r[8 * j + 7]));
      }
    }
  }
  if (row_ok) *lse_dst = p.visit_fold ? mw.lse : lse_t;
}

template <int D>
__device__ void softmax_role(const FwdParams& p, const FwdBars& br, uint32_t tmem, int w,
                             const Ctl& cx) {
  const int t = threadIdx.x - w * 128;            // row inside the query tile
  const int quarter = (threadIdx.x >> 5) & 3;     // TMEM lane quarter of this warp
  const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t tS = tmem + lane_off + w * 128;  // S (fp32) and P (bf16 pairs, first 64 cols)
  const uint32_t tO = tmem + lane_off + 256 + w * 128;
  const float c2 = p.scale_log2;
  uint32_t s_phase = 0u, units_w = 0u;

  for (int k = 0;; ++k) {
    int u;
    const bool got = next_unit(br, k, cx, u);
    if (!__all_sync(0xffffffffu, got)) return;
    u = __shfl_sync(0xffffffffu, u, 0);
    if (u < 0) break;
    const Unit x = decode_unit(p, u);
    if (w == 1 && !x.valid1) continue;
    const int qt = w ? x.qt[1] : x.qt[0];
    const int h = w ? x.h[1] : x.h[0];
    const int qrow = qt * BM + t;                  // row inside the ring block
    // running max m (log2 units) and row sum l of P
    float m = -INFINITY, l = 0.f;
    KvIter it;
    it.start(p, x);

    for (int idx = 0; idx < x.n_kv; ++idx, it.next(p)) {
      // keys allowed for this row: columns 0..lim of the tile.  Warp-uniform
      // `masked`: both exp_row_store instantiations issue warp-collective
      // tcgen05.st, which all 32 lanes must execute together; lanes whose own
      // row needs no mask (lim = 127) run the masked code harmlessly.
      int lim = min(BN, p.blk_len - it.kl * BN) - 1;
      if (p.causal && it.jb == x.blk) lim = min(lim, qrow - it.kl * BN - p.diag_shift);
      const bool masked = __any_sync(0xffffffffu, lim < BN - 1);
      if (p.o_acc != nullptr && p.visit_fold && idx == x.n_kv - 1 && qrow < p.blk_len) {
        // the epilogue reads this row of the running accumulator (D fp32) back
        const char* a = reinterpret_cast<const char*>(
            p.o_acc + ((static_cast<long long>(x.b) * p.L + qrow) * p.Hq + h) * D);
#pragma unroll
        for (int c = 0; c < D * 4; c += 128) prefetch_l2(a + c);
      }

      bool ok = wait_bar(br.s_full(w), s_phase, cx, SITE_S_FULL);
      if (!__all_sync(0xffffffffu, ok)) return;
      s_phase ^= 1u;
      tc_fence_after();

      // S in two halves: the max over the first 64 columns runs while the
      // second half is still being read from TMEM
      uint32_t sr[128];
      tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_wait_ld();
      tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
      tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
      if (masked) {
#pragma unroll
        for (int j = 0; j < 64; ++j)
          if (j > lim) sr[j] = __float_as_uint(-INFINITY);
      }
      float mx[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx[i] = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; ++j)
        mx[j & 7] = fmax3(mx[j & 7], __uint_as_float(sr[2 * j]), __uint_as_float(sr[2 * j + 1]));
      tmem_wait_ld();
      if (masked) {
#pragma unroll
        for (int j = 64; j < 128; ++j)
          if (j > lim) sr[j] = __float_as_uint(-INFINITY);
      }
#pragma unroll
      for (int j = 32; j < 64; ++j)
        mx[j & 7] = fmax3(mx[j & 7], __uint_as_float(sr[2 * j]), __uint_as_float(sr[2 * j + 1]));
      const float rmax = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                               fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      const float m_tile = (rmax == -INFINITY) ? -INFINITY : rmax * c2;
      // Rescale when the tile maximum exceeds the reference by more than
      // RESCALE_LOG2 (the decision is per row; the O round trip in TMEM runs
      // for the warp when any of its rows needs it, with alpha = 1 for the
      // others; the final O / l cancels the reference exactly).
      const bool need = m_tile > m + RESCALE_LOG2;
      float alpha = 1.f;
      if (__any_sync(0xffffffffu, need)) {
        const float m_new = need ? m_tile : m;
        alpha = (m_new == m) ? 1.f : ex2_approx(m - m_new);
        if (idx > 0) {
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
      }
      const float rsum = masked ? exp_row_store<true>(sr, c2, m, lim, tS, br.p_half(w))
                                : exp_row_store<false>(sr, c2, m, lim, tS, br.p_half(w));
      l = l * alpha + rsum;
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
      if (p.o_acc != nullptr) {
        // a row with no allowed key (strict diagonal, row 0) is an empty
        // partial: o = 0, lse = -inf, which the fold ignores
        visit_epilogue<D>(p, tO, row_ok, x.b, pos, h, l > 0.f ? inv_l : 0.f, (m + log2f(l)) * LN2);
        tc_fence_before();
        mbar_arrive(br.o_free(w));
        ++units_w;
        continue;
      }
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

  FwdBars br;
  br.layout(base + C::OFF_BAR, C::NS, base + C::OFF_UNITS);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(base_ptr + C::OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(base_ptr + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    br.init(C::NS);
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
  const Ctl cx{abort_flag, p.wait_limit_ns, &g_ra_status};

  if (warp < 8) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" :: "n"(SOFTMAX_REGS));
    softmax_role<D>(p, br, tmem, warp >> 2, cx);
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" :: "n"(CONTROL_REGS));
    if (warp == WARP_LOAD) {
      fwd_loader_role<Bf16Geom<D>>(p, br, base, cx);
    } else if (warp == WARP_MMA) {
      fwd_mma_role<Bf16Geom<D>>(p, br, base, tmem, cx);
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

cudaError_t next_ticket_counter(cudaStream_t stream, unsigned int** counter) {
  static std::atomic<unsigned> next{0u};
  void* base = nullptr;
  cudaError_t e = symbol_address(reinterpret_cast<const void*>(&g_ra_tickets), &base, stream);
  if (e != cudaSuccess) return e;
  unsigned int* slot = static_cast<unsigned int*>(base) + (next.fetch_add(1u) % kTicketSlots);
  e = cudaMemsetAsync(slot, 0, sizeof(unsigned int), stream);
  if (e != cudaSuccess) return e;
  *counter = slot;
  return cudaSuccess;
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
