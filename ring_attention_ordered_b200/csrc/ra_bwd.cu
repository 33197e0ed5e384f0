// Backward pass of ring-ordered blockwise attention for sm_100a.
//
// What it computes: the gradients of the forward pass for an upstream
// gradient dO, recomputing the attention weights from the stored logsumexp
// instead of storing them (FlashAttention article, section 二: 核心原理 and
// 重计算 -- only O and the softmax statistics are kept):
//   P  = exp(scale * Q K^T - lse)          (per query row; masked entries 0)
//   dV = P^T dO
//   dP = dO V^T,  D = rowsum(dO * O),  dS = P * (dP - D)
//   dQ = scale * dS K,  dK = scale * dS^T Q
// (D equals rowsum(P * dP), the row term of the softmax Jacobian, because
// O = P V.)  Grouped-query heads (lnwmold page §2.2) add their dK, dV into the
// shared K/V head.  The work is ordered as the ring of "Ring Attention 环注意力"
// (L4 §4.2): the query block of host i visits K/V blocks (i - t) mod N, and
// the K/V block of host j visits query blocks (j + t) mod N -- the order in
// which dK_j, dV_j would travel the ring; causal visits with a later K/V block
// are skipped (L4 §4.5 limitation 2).
//
// How (B200 design): two persistent kernels, one CTA per SM, each with two
// softmax warpgroups (warps 0-7; both cover all 128 TMEM lanes, one tile row
// per lane, and split the tile's 128 columns), a TMA loader warp (8) and a
// tcgen05.mma warp (9).
//   * ra_bwd_dq_kernel: a unit is one 128-row query tile of one head; it
//     computes D for its rows (written to the workspace), then for every K/V
//     tile S = Q K^T and dP = dO V^T into TMEM, P and dS in the softmax
//     warps (dS as bf16 over dP), and dQ += dS K accumulated in TMEM.  S is
//     released as soon as it is read, so the next tile's S overlaps the
//     exponentials; K (read early by S and late by dQ) has three stages.
//   * ra_bwd_dkdv_kernel (after it, on the same stream): a unit is one
//     128-key tile of one K/V head; for every query tile of every head of the
//     group, S^T = K Q^T and dP^T = V dO^T into TMEM; the softmax warps read
//     S^T (released at once, so the next tile's S^T overlaps them), form P^T,
//     read dP^T and write P^T and dS^T as bf16 over it; dV += P^T dO and
//     dK += dS^T Q accumulate in TMEM: no atomics, every gradient is written
//     once.  Q (read early by S^T and late by dK) has three stages.
//   P is rounded to bf16 once and that value feeds both dV and dS.
//   The CTAs of each launch take their units from one work queue
//   (ra_unit_queue.cuh), head by head and longest first inside a head, so
//   they stay within about one unit of each other and share K/V (dQ kernel)
//   or Q/dO tiles (dK/dV kernel) in L2.
//   Every mbarrier wait is bounded (ra_sync.cuh).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "ptx_sm100.cuh"
#include "ra_internal.h"
#include "ra_sync.cuh"
#include "ra_unit_queue.cuh"
#include "ring_attn.h"

namespace ra {
namespace bwd {

constexpr int TM = 128;              // rows per tile (queries or keys)
constexpr int BOX_COLS = 64;
constexpr int BOX_BYTES = 128 * 128;
// Two softmax warpgroups split each tile's 128 columns (64 each; both cover
// all 128 TMEM lanes, so every SM sub-partition runs two of their warps and
// one hides the other's TMEM and MUFU latency), then the loader and MMA warps.
constexpr int NUM_THREADS = 320;
constexpr int SOFTMAX_THREADS = 256;
constexpr int WARP_LOAD = 8;
constexpr int WARP_MMA = 9;
constexpr int HALF = 64;             // columns per softmax warpgroup
constexpr float LOG2E = 1.4426950408889634f;


// Device status word of the backward kernels: 0 = ok, else (code << 32) | where.
__device__ unsigned long long g_status = 0ull;

enum Site : uint32_t {
  SITE_KV_FULL = 17, SITE_KV_EMPTY, SITE_QD_FULL, SITE_QD_EMPTY, SITE_S_FULL, SITE_S_FREE,
  SITE_DP_FULL, SITE_P_FULL, SITE_DS_FULL, SITE_ACC_DONE, SITE_ACC_FREE, SITE_UNIT
};

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// S-like MMA over the head dimension (A, B both K-major): D/16 steps.
template <int KK>
struct KStep {
  static constexpr uint32_t OFF = ((KK / 4) * BOX_BYTES + (KK % 4) * 32) >> 4;
};
template <int D>
__device__ __forceinline__ void mma_kmajor(uint32_t d, uint32_t a, uint32_t b, uint32_t hi,
                                           uint32_t idesc) {
  if (elect_one()) mma_ss<KStep<0>::OFF, KStep<0>::OFF>(d, a, hi, b, hi, idesc, 0u);
  if (elect_one()) mma_ss<KStep<1>::OFF, KStep<1>::OFF>(d, a, hi, b, hi, idesc, 1u);
  if (elect_one()) mma_ss<KStep<2>::OFF, KStep<2>::OFF>(d, a, hi, b, hi, idesc, 1u);
  if (elect_one()) mma_ss<KStep<3>::OFF, KStep<3>::OFF>(d, a, hi, b, hi, idesc, 1u);
  if constexpr (D == 128) {
    if (elect_one()) mma_ss<KStep<4>::OFF, KStep<4>::OFF>(d, a, hi, b, hi, idesc, 1u);
    if (elect_one()) mma_ss<KStep<5>::OFF, KStep<5>::OFF>(d, a, hi, b, hi, idesc, 1u);
    if (elect_one()) mma_ss<KStep<6>::OFF, KStep<6>::OFF>(d, a, hi, b, hi, idesc, 1u);
    if (elect_one()) mma_ss<KStep<7>::OFF, KStep<7>::OFF>(d, a, hi, b, hi, idesc, 1u);
  }
}

// Accumulating MMA with A (bf16 pairs, 128 along K) in TMEM and B MN-major in
// shared memory (K = 128 rows of 128 bytes per 64-column box): 8 steps of
// 16, B advancing 16 rows (2048 bytes) per step.  A was written by the two
// softmax warpgroups into their own halves of a 128-column TMEM region: K
// rows 0-63 as pairs at columns 0-31 of the region, rows 64-127 at 64-95.
__device__ __forceinline__ void mma_tmem_a_split(uint32_t d, uint32_t a_tmem, uint32_t b,
                                                 uint32_t hi, uint32_t idesc, uint32_t acc) {
  if (elect_one()) mma_ts<0, 0>(d, a_tmem, b, hi, idesc, acc);
  if (elect_one()) mma_ts<8, 128>(d, a_tmem, b, hi, idesc, 1u);
  if (elect_one()) mma_ts<16, 256>(d, a_tmem, b, hi, idesc, 1u);
  if (elect_one()) mma_ts<24, 384>(d, a_tmem, b, hi, idesc, 1u);
  if (elect_one()) mma_ts<64, 512>(d, a_tmem, b, hi, idesc, 1u);
  if (elect_one()) mma_ts<72, 640>(d, a_tmem, b, hi, idesc, 1u);
  if (elect_one()) mma_ts<80, 768>(d, a_tmem, b, hi, idesc, 1u);
  if (elect_one()) mma_ts<88, 896>(d, a_tmem, b, hi, idesc, 1u);
}

__device__ __forceinline__ void commit(uint32_t bar) {
  if (elect_one()) tc_commit(bar);
}

// Store one row of fp32 accumulator columns [col0, col0 + D) of TMEM, times
// `mul`, as bf16 to dst (D contiguous elements); all lanes load, only
// `valid` lanes store.
template <int D>
__device__ __forceinline__ void store_acc_row(uint32_t taddr, float mul, __nv_bfloat16* dst,
                                              bool valid) {
#pragma unroll
  for (int cc = 0; cc < D / 32; ++cc) {
    uint32_t o[32];
    tmem_ld32(taddr + cc * 32, o);
    tmem_wait_ld();
    uint32_t pk[16];
#pragma unroll
    for (int j = 0; j < 16; ++j)
      pk[j] = pack_bf16x2(__uint_as_float(o[2 * j]) * mul, __uint_as_float(o[2 * j + 1]) * mul);
    if (valid) {
      uint4* d4 = reinterpret_cast<uint4*>(dst + cc * 32);
#pragma unroll
      for (int j = 0; j < 4; ++j) d4[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
    }
  }
}

// Per-visit form of store_acc_row: the row (times `mul`) is written to, or
// with `fold` added to, the fp32 accumulator row acc (D floats); `dst`, if
// not null, receives the bf16 rounding of the new accumulator row.
template <int D>
__device__ __forceinline__ void fold_acc_row(uint32_t taddr, float mul, float* acc, bool fold,
                                             __nv_bfloat16* dst, bool valid) {
#pragma unroll
  for (int cc = 0; cc < D / 32; ++cc) {
    uint32_t o[32];
    tmem_ld32(taddr + cc * 32, o);
    tmem_wait_ld();
    if (valid) {
      float4* a4 = reinterpret_cast<float4*>(acc + cc * 32);
      float r[32];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float4 x = make_float4(__uint_as_float(o[4 * j]) * mul, __uint_as_float(o[4 * j + 1]) * mul,
                               __uint_as_float(o[4 * j + 2]) * mul,
                               __uint_as_float(o[4 * j + 3]) * mul);
        if (fold) {
          const float4 a = a4[j];
          x.x += a.x;
          x.y += a.y;
          x.z += a.z;
          x.w += a.w;
        }
        a4[j] = x;
        r[4 * j] = x.x;
        r[4 * j + 1] = x.y;
        r[4 * j + 2] = x.z;
        r[4 * j + 3] = x.w;
      }
      if (dst != nullptr) {
        uint4* d4 = reinterpret_cast<uint4*>(dst + cc * 32);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          d4[j] = make_uint4(pack_bf16x2(r[8 * j], r[8 * j + 1]), pack_bf16x2(r[8 * j + 2], r[8 * j + 3]),
                             pack_bf16x2(r[8 * j + 4], r[8 * j + 5]),
                             pack_bf16x2(r[8 * j + 6], r[8 * j + 7]));
      }
    }
  }
}

// dS over 32 columns: ds = p * (dp - D), p from bf16 pairs pk (16 words), dp
// from TMEM (fp32), D per column (dkdv: one per query, from shared memory)
// or one for the whole row (dq: the row's own D).
template <bool PER_COLUMN>
__device__ __forceinline__ void ds_chunk(const uint32_t (&pk)[16], const uint32_t (&dp)[32],
                                         const float* dcol, float drow, uint32_t (&out)[16]) {
  const uint64_t dr2 = f2_pack(drow, drow);
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const uint64_t p2 = f2_pack(bf16lo(pk[j]), bf16hi(pk[j]));
    const uint64_t dd = PER_COLUMN ? f2_pack(dcol[2 * j], dcol[2 * j + 1]) : dr2;
    const uint64_t d2 =
        f2_sub(f2_pack(__uint_as_float(dp[2 * j]), __uint_as_float(dp[2 * j + 1])), dd);
    float a, b;
    f2_unpack(f2_mul(p2, d2), a, b);
    out[j] = pack_bf16x2(a, b);
  }
}

// =====================================================================
// dQ kernel: query-stationary
// =====================================================================
template <int D>
struct QCfg {
  static constexpr int TILE = TM * D * 2;
  // K tiles are read by S (early in a step) and by dQ (late), V tiles only by
  // dP: three K stages let the next-but-one K tile load while dQ still reads
  // the current one, two V stages suffice
  static constexpr int NK = (D == 128) ? 3 : 6;
  static constexpr int NV = (D == 128) ? 2 : 4;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = TILE;
  static constexpr int OFF_K = 2 * TILE;
  static constexpr int OFF_V = OFF_K + NK * TILE;
  static constexpr int OFF_BAR = OFF_V + NV * TILE;
  // qo_full, qo_empty, k_full[NK], k_empty[NK], v_full[NV], v_empty[NV],
  // s_full, s_free, dp_full, ds_full, acc_done, acc_free, drain, then the
  // unit queue's barriers
  static constexpr int NUM_BARS = 2 + 2 * NK + 2 * NV + 7 + UNIT_QUEUE_DEPTH;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_UNITS = OFF_MISC + 16;
  static constexpr int SMEM_BYTES = OFF_UNITS + 4 * UNIT_QUEUE_DEPTH + 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct QBars {
  uint32_t base;
  int nk, nv;
  __device__ __forceinline__ uint32_t qo_full() const { return base; }
  __device__ __forceinline__ uint32_t qo_empty() const { return base + 8; }
  __device__ __forceinline__ uint32_t k_full(int s) const { return base + 16 + 8u * s; }
  __device__ __forceinline__ uint32_t k_empty(int s) const { return base + 16 + 8u * (nk + s); }
  __device__ __forceinline__ uint32_t v_full(int s) const { return base + 16 + 16u * nk + 8u * s; }
  __device__ __forceinline__ uint32_t v_empty(int s) const {
    return base + 16 + 16u * nk + 8u * (nv + s);
  }
  __device__ __forceinline__ uint32_t s_full() const { return base + 16 + 16u * nk + 16u * nv; }
  __device__ __forceinline__ uint32_t s_free() const { return s_full() + 8; }
  __device__ __forceinline__ uint32_t dp_full() const { return s_full() + 16; }
  __device__ __forceinline__ uint32_t ds_full() const { return s_full() + 24; }
  __device__ __forceinline__ uint32_t acc_done() const { return s_full() + 32; }
  __device__ __forceinline__ uint32_t acc_free() const { return s_full() + 40; }
  __device__ __forceinline__ uint32_t drain() const { return s_full() + 48; }
  __device__ __forceinline__ uint32_t units0() const { return s_full() + 56; }
};

struct QUnit {
  int b, h, blk, qt, n;
};

// Units in (batch, head) order, longest first inside a head: the query block
// i from last to first, its tiles from last to first.
__device__ __forceinline__ QUnit q_unit(const BwdParams& p, int u) {
  const int per_head = p.n_ring * p.tiles_per_blk;
  const int bh = u / per_head;
  const int rem = u - bh * per_head;
  QUnit x;
  x.b = bh / p.Hq;
  x.h = bh - x.b * p.Hq;
  x.blk = p.n_ring - 1 - rem / p.tiles_per_blk;
  x.qt = p.tiles_per_blk - 1 - rem % p.tiles_per_blk;
  x.n = p.causal ? (x.blk * p.tiles_per_blk + x.qt + 1) : p.n_ring * p.tiles_per_blk;
  return x;
}

// K/V tiles of a query unit in ring order: own block first (tiles 0..qt
// under causal masking), then blocks blk-1, blk-2, ... wrapping around.
struct KvWalk {
  int jb, kl, end;
  __device__ __forceinline__ void start(const BwdParams& p, const QUnit& x) {
    jb = x.blk;
    kl = 0;
    end = p.causal ? x.qt + 1 : p.tiles_per_blk;
  }
  __device__ __forceinline__ void next(const BwdParams& p) {
    if (++kl == end) {
      kl = 0;
      jb = (jb == 0) ? p.n_ring - 1 : jb - 1;
      end = p.tiles_per_blk;
    }
  }
};

template <int D>
__device__ void dq_loader(const BwdParams& p, const QBars& br, const UnitQueue& uq, uint32_t base,
                          const Ctl& cx) {
  using C = QCfg<D>;
  constexpr int NBOX = D / BOX_COLS;
  uint32_t kv_it = 0, units = 0;
  bool qo_pending = false;
  for (int k = 0;; ++k) {
    const int u = uq.take(p.tickets_dq, p.units_dq, k);
    if (u < 0) break;
    const QUnit x = q_unit(p, u);
    if (units > 0 && !wait_warp(br.qo_empty(), (units - 1) & 1u, cx, SITE_QD_EMPTY)) goto drain;
    if ((p.debug_flags & 1u) && units == 0) {
      // fault injection: the first query tiles are never requested
    } else {
      const int row = x.b * p.L + x.blk * p.blk_len + x.qt * TM;
      if (elect_one()) {
        mbar_arrive_expect_tx(br.qo_full(), 2 * C::TILE);
#pragma unroll
        for (int bx = 0; bx < NBOX; ++bx) {
          tma_load_3d(base + C::OFF_Q + bx * BOX_BYTES, &p.tm_q, br.qo_full(), bx * BOX_COLS, x.h, row);
          tma_load_3d(base + C::OFF_DO + bx * BOX_BYTES, &p.tm_do, br.qo_full(), bx * BOX_COLS, x.h,
                      row);
        }
      }
      __syncwarp();
      qo_pending = true;
    }
    ++units;
    KvWalk it;
    it.start(p, x);
    const int kvh = x.h / p.group;
    for (int idx = 0; idx < x.n; ++idx, it.next(p)) {
      const int row = x.b * p.L + it.jb * p.blk_len + it.kl * TM;
      const int sk = kv_it % C::NK, sv = kv_it % C::NV;
      if (!wait_warp(br.k_empty(sk), ((kv_it / C::NK) & 1u) ^ 1u, cx, SITE_KV_EMPTY)) goto drain;
      if (elect_one()) {
        mbar_arrive_expect_tx(br.k_full(sk), C::TILE);
#pragma unroll
        for (int bx = 0; bx < NBOX; ++bx)
          tma_load_3d(base + C::OFF_K + sk * C::TILE + bx * BOX_BYTES, &p.tm_k, br.k_full(sk),
                      bx * BOX_COLS, kvh, row);
      }
      __syncwarp();
      if (!wait_warp(br.v_empty(sv), ((kv_it / C::NV) & 1u) ^ 1u, cx, SITE_KV_EMPTY)) goto drain;
      if (elect_one()) {
        mbar_arrive_expect_tx(br.v_full(sv), C::TILE);
#pragma unroll
        for (int bx = 0; bx < NBOX; ++bx)
          tma_load_3d(base + C::OFF_V + sv * C::TILE + bx * BOX_BYTES, &p.tm_v, br.v_full(sv),
                      bx * BOX_COLS, kvh, row);
      }
      __syncwarp();
      ++kv_it;
    }
  }
  return;
drain:
  if ((threadIdx.x & 31) == 0) {
    // let the copies already issued land before the CTA's shared memory goes
    const uint32_t nk = kv_it < static_cast<uint32_t>(C::NK) ? kv_it : C::NK;
    for (uint32_t i = 0; i < nk; ++i) {
      const uint32_t it = kv_it - 1 - i;
      drain_wait(br.k_full(it % C::NK), (it / C::NK) & 1u, 200000000ull);
    }
    const uint32_t nv = kv_it < static_cast<uint32_t>(C::NV) ? kv_it : C::NV;
    for (uint32_t i = 0; i < nv; ++i) {
      const uint32_t it = kv_it - 1 - i;
      drain_wait(br.v_full(it % C::NV), (it / C::NV) & 1u, 200000000ull);
    }
    if (qo_pending) drain_wait(br.qo_full(), (units - 1) & 1u, 200000000ull);
  }
  __syncwarp();
}

template <int D>
__device__ void dq_mma(const BwdParams& p, const QBars& br, const UnitQueue& uq, uint32_t base,
                       uint32_t tmem, const Ctl& cx) {
  using C = QCfg<D>;
  constexpr uint32_t IDESC_S = idesc_bf16_f32(TM, TM, false);
  constexpr uint32_t IDESC_DQ = idesc_bf16_f32(TM, D, true);
  const uint64_t dq0 = smem_desc_sw128(base + C::OFF_Q, 16, 1024);
  const uint64_t ddo0 = smem_desc_sw128(base + C::OFF_DO, 16, 1024);
  const uint64_t dk0 = smem_desc_sw128(base + C::OFF_K, 16, 1024);
  const uint64_t dv0 = smem_desc_sw128(base + C::OFF_V, 16, 1024);
  const uint64_t dkmn0 = smem_desc_sw128(base + C::OFF_K, BOX_BYTES, 1024);
  const uint32_t q_lo = static_cast<uint32_t>(dq0), do_lo = static_cast<uint32_t>(ddo0);
  const uint32_t k_lo = static_cast<uint32_t>(dk0), v_lo = static_cast<uint32_t>(dv0);
  const uint32_t kmn_lo = static_cast<uint32_t>(dkmn0);
  const uint32_t hi = static_cast<uint32_t>(dk0 >> 32), mn_hi = static_cast<uint32_t>(dkmn0 >> 32);
  const uint32_t t_s = tmem, t_dp = tmem + 128, t_dq = tmem + 256;
  uint32_t kv_it = 0, units = 0, step = 0;
  // S = Q K^T from K stage sk, dP = dO V^T from V stage sv (all K-major)
  auto issue_s = [&](int sk) { mma_kmajor<D>(t_s, q_lo, k_lo + ((sk * C::TILE) >> 4), hi, IDESC_S); };
  auto issue_dp = [&](int sv) {
    mma_kmajor<D>(t_dp, do_lo, v_lo + ((sv * C::TILE) >> 4), hi, IDESC_S);
  };
  for (int k = 0;; ++k) {
    int u;
    if (!uq.read(k, cx, SITE_UNIT, u)) goto drain;
    if (u < 0) break;
    const QUnit x = q_unit(p, u);
    const int n = x.n;
    if (!wait_warp(br.qo_full(), units & 1u, cx, SITE_QD_FULL)) goto drain;
    {
      const int sk = kv_it % C::NK, sv = kv_it % C::NV;
      if (!wait_warp(br.k_full(sk), (kv_it / C::NK) & 1u, cx, SITE_KV_FULL)) goto drain;
      tc_fence_after();
      issue_s(sk);
      commit(br.s_full());
      if (!wait_warp(br.v_full(sv), (kv_it / C::NV) & 1u, cx, SITE_KV_FULL)) goto drain;
      tc_fence_after();
      issue_dp(sv);
      commit(br.dp_full());
      commit(br.v_empty(sv));
    }
    for (int idx = 0; idx < n; ++idx) {
      const bool more = idx + 1 < n;
      const int sk = kv_it % C::NK;
      const int sk1 = (kv_it + 1) % C::NK, sv1 = (kv_it + 1) % C::NV;
      if (more) {
        // S for the next K/V tile as soon as the softmax has read this one
        if (!wait_warp(br.s_free(), step & 1u, cx, SITE_S_FREE)) goto drain;
        if (!wait_warp(br.k_full(sk1), ((kv_it + 1) / C::NK) & 1u, cx, SITE_KV_FULL)) goto drain;
        tc_fence_after();
        issue_s(sk1);
        commit(br.s_full());
      }
      if (!wait_warp(br.ds_full(), step & 1u, cx, SITE_DS_FULL)) goto drain;
      if (idx == 0 && units > 0 &&
          !wait_warp(br.acc_free(), (units - 1) & 1u, cx, SITE_ACC_FREE))
        goto drain;
      tc_fence_after();
      mma_tmem_a_split(t_dq, t_dp, kmn_lo + ((sk * C::TILE) >> 4), mn_hi, IDESC_DQ,
                       idx > 0 ? 1u : 0u);
      commit(br.k_empty(sk));
      if (more) {
        if (!wait_warp(br.v_full(sv1), ((kv_it + 1) / C::NV) & 1u, cx, SITE_KV_FULL)) goto drain;
        tc_fence_after();
        issue_dp(sv1);
        commit(br.dp_full());
        commit(br.v_empty(sv1));
      }
      ++step;
      ++kv_it;
    }
    commit(br.acc_done());
    commit(br.qo_empty());
    ++units;
  }
  return;
drain:
  commit(br.drain());
  if ((threadIdx.x & 31) == 0) drain_wait(br.drain(), 0u, 200000000ull);
  __syncwarp();
}

template <int D>
__device__ void dq_softmax(const BwdParams& p, const QBars& br, const UnitQueue& uq, uint32_t tmem,
                           int wg, const Ctl& cx) {
  constexpr int D2 = D / 2;                        // dQ columns of this warpgroup
  const int t = threadIdx.x & 127;                 // row inside the query tile
  const int quarter = (threadIdx.x >> 5) & 3;
  const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
  // this warpgroup's keys: columns [64 wg, 64 wg + 64) of S and of dP
  const uint32_t t_s = tmem + lane_off + HALF * wg, t_dp = tmem + lane_off + 128 + HALF * wg;
  const uint32_t t_dq = tmem + lane_off + 256 + D2 * wg;
  const int col0 = HALF * wg;
  const float c2 = p.scale_log2;
  uint32_t units = 0, step = 0;
  for (int k = 0;; ++k) {
    int u;
    if (!uq.read(k, cx, SITE_UNIT, u)) return;
    if (u < 0) break;
    const QUnit x = q_unit(p, u);
    const int qrow = x.qt * TM + t;
    const bool valid = qrow < p.blk_len;
    const long long grow = static_cast<long long>(x.blk) * p.blk_len + qrow;
    const long long vidx = (static_cast<long long>(x.b) * p.Hq + x.h) * p.L + grow;
    // D = rowsum(dO * O) of this row (both warpgroups form it; the first
    // stores it), and the row's lse in base 2
    float dvec = 0.f, nlse2 = -INFINITY;
    if (valid) {
      const long long off = ((static_cast<long long>(x.b) * p.L + grow) * p.Hq + x.h) * D;
      const uint4* o4 = reinterpret_cast<const uint4*>(p.out + off);
      const uint4* g4 = reinterpret_cast<const uint4*>(p.dout + off);
      float acc = 0.f;
#pragma unroll 4
      for (int j = 0; j < D / 8; ++j) {
        const uint4 a = o4[j], g = g4[j];
        acc = fmaf(bf16lo(a.x), bf16lo(g.x), acc);
        acc = fmaf(bf16hi(a.x), bf16hi(g.x), acc);
        acc = fmaf(bf16lo(a.y), bf16lo(g.y), acc);
        acc = fmaf(bf16hi(a.y), bf16hi(g.y), acc);
        acc = fmaf(bf16lo(a.z), bf16lo(g.z), acc);
        acc = fmaf(bf16hi(a.z), bf16hi(g.z), acc);
        acc = fmaf(bf16lo(a.w), bf16lo(g.w), acc);
        acc = fmaf(bf16hi(a.w), bf16hi(g.w), acc);
      }
      dvec = acc;
      if (wg == 0) p.dvec[vidx] = acc;
      nlse2 = -p.lse[vidx] * LOG2E;
    }
    const uint64_t nl2 = f2_pack(nlse2, nlse2);
    const uint64_t c2x2 = f2_pack(c2, c2);

    KvWalk it;
    it.start(p, x);
    for (int idx = 0; idx < x.n; ++idx, it.next(p)) {
      // keys allowed for this row: tile columns 0..lim
      int lim = min(TM, p.blk_len - it.kl * TM) - 1;
      if (p.causal && it.jb == x.blk) lim = min(lim, qrow - it.kl * TM - p.diag_shift);
      const int lim_local = lim - col0;
      const bool masked = __any_sync(0xffffffffu, lim_local < HALF - 1);
      if (!wait_warp(br.s_full(), step & 1u, cx, SITE_S_FULL)) return;
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld32(t_s, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(t_s + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(br.s_free());
      // P = 2^(s * scale * log2 e - lse * log2 e), rounded to bf16 pairs
      uint32_t pk[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const uint64_t x2 =
            f2_fma(f2_pack(__uint_as_float(sr[2 * j]), __uint_as_float(sr[2 * j + 1])), c2x2, nl2);
        float p0, p1;
        f2_unpack(x2, p0, p1);
        p0 = ex2_approx(p0);
        p1 = ex2_approx(p1);
        if (masked) {
          p0 = (2 * j > lim_local) ? 0.f : p0;
          p1 = (2 * j + 1 > lim_local) ? 0.f : p1;
        }
        pk[j] = pack_bf16x2(p0, p1);
      }
      if (!wait_warp(br.dp_full(), step & 1u, cx, SITE_DP_FULL)) return;
      tc_fence_after();
      // dS = P (dP - D) in two chunks of 32 keys, each stored as 16 columns of
      // bf16 pairs over this warpgroup's dP columns that have been read
      {
        // both 32-key chunks of dP are read before any dS pair overwrites them
        uint32_t dp[2][32];
        tmem_ld32(t_dp, dp[0]);
        tmem_ld32(t_dp + 32, dp[1]);
        tmem_wait_ld();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t ds[16];
          ds_chunk<false>(*reinterpret_cast<const uint32_t(*)[16]>(&pk[16 * cc]), dp[cc], nullptr,
                          dvec, ds);
          tmem_st16(t_dp + 16 * cc, ds);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(br.ds_full());
      ++step;
    }
    // epilogue: dQ = scale * (dS K) accumulated in TMEM, half the columns
    if (!wait_warp(br.acc_done(), units & 1u, cx, SITE_ACC_DONE)) return;
    tc_fence_after();
    const long long qoff = ((static_cast<long long>(x.b) * p.L + grow) * p.Hq + x.h) * D + D2 * wg;
    if (p.dq_acc != nullptr)
      fold_acc_row<D2>(t_dq, p.scale, p.dq_acc + qoff, p.fold_q, p.dq ? p.dq + qoff : nullptr,
                       valid);
    else
      store_acc_row<D2>(t_dq, p.scale, p.dq + qoff, valid);
    tc_fence_before();
    mbar_arrive(br.acc_free());
    ++units;
  }
}

template <int D>
__global__ void __launch_bounds__(NUM_THREADS, 1) ra_bwd_dq_kernel(const __grid_constant__ BwdParams p) {
  using C = QCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gen = smem_raw + (base - raw);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(gen + C::OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(gen + C::OFF_MISC + 4);
  const QBars br{base + C::OFF_BAR, C::NK, C::NV};
  // the loader runs at most two units ahead of the softmax warpgroups (it
  // takes unit k + 2 only after the MMA warp has finished unit k's products,
  // which needed all of unit k's dS), so the queue's four slots never overrun
  const UnitQueue uq{br.units0(), base + C::OFF_UNITS};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0 && lane == 0) {
    mbar_init(br.qo_full(), 1);
    mbar_init(br.qo_empty(), 1);
    for (int s = 0; s < C::NK; ++s) {
      mbar_init(br.k_full(s), 1);
      mbar_init(br.k_empty(s), 1);
    }
    for (int s = 0; s < C::NV; ++s) {
      mbar_init(br.v_full(s), 1);
      mbar_init(br.v_empty(s), 1);
    }
    mbar_init(br.s_full(), 1);
    mbar_init(br.s_free(), SOFTMAX_THREADS);
    mbar_init(br.dp_full(), 1);
    mbar_init(br.ds_full(), SOFTMAX_THREADS);
    mbar_init(br.acc_done(), 1);
    mbar_init(br.acc_free(), SOFTMAX_THREADS);
    mbar_init(br.drain(), 1);
    uq.init();
    *abort_flag = 0u;
    fence_mbarrier_init();
  }
  if (warp == WARP_LOAD && lane == 0) {
    prefetch_tensormap(&p.tm_q);
    prefetch_tensormap(&p.tm_do);
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
  const Ctl cx{abort_flag, p.wait_limit_ns, &g_status};
  if (warp < 8) {
    dq_softmax<D>(p, br, uq, tmem, warp >> 2, cx);
  } else if (warp == WARP_LOAD) {
    dq_loader<D>(p, br, uq, base, cx);
  } else {
    dq_mma<D>(p, br, uq, base, tmem, cx);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// =====================================================================
// dK/dV kernel: key-stationary
// =====================================================================
template <int D>
struct KCfg {
  static constexpr int TILE = TM * D * 2;
  // Q tiles are read by S^T early in a step (the next tile's S^T overlaps the
  // current exponentials) and by dK late, so Q needs three stages; dO is read
  // by dP^T and dV within one step, two stages
  static constexpr int NQ = (D == 128) ? 3 : 6;
  static constexpr int NO = (D == 128) ? 2 : 4;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = TILE;
  static constexpr int OFF_Q = 2 * TILE;
  static constexpr int OFF_DO = OFF_Q + NQ * TILE;
  static constexpr int OFF_LSE = OFF_DO + NO * TILE;    // per Q stage: -lse*log2e [128]
  static constexpr int OFF_DV = OFF_LSE + NQ * TM * 4;  // per dO stage: D [128]
  static constexpr int OFF_BAR = OFF_DV + NO * TM * 4;
  // kv_full, kv_empty, q_full[NQ], q_empty[NQ], do_full[NO], do_empty[NO],
  // s_full, dp_full, s_free, pd_full, acc_done, acc_free, drain, then the
  // unit queue's barriers
  static constexpr int NUM_BARS = 2 + 2 * NQ + 2 * NO + 7 + UNIT_QUEUE_DEPTH;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_UNITS = OFF_MISC + 16;
  // no alignment slack: the kernel checks that the dynamic shared memory
  // starts on a 1024-byte boundary (the 128-byte swizzle needs it) and
  // reports RA_ERR_UNSUPPORTED otherwise
  static constexpr int SMEM_BYTES = OFF_UNITS + 4 * UNIT_QUEUE_DEPTH;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct KBars {
  uint32_t base;
  int nq, no;
  __device__ __forceinline__ uint32_t kv_full() const { return base; }
  __device__ __forceinline__ uint32_t kv_empty() const { return base + 8; }
  __device__ __forceinline__ uint32_t q_full(int s) const { return base + 16 + 8u * s; }
  __device__ __forceinline__ uint32_t q_empty(int s) const { return base + 16 + 8u * (nq + s); }
  __device__ __forceinline__ uint32_t do_full(int s) const { return base + 16 + 16u * nq + 8u * s; }
  __device__ __forceinline__ uint32_t do_empty(int s) const {
    return base + 16 + 16u * nq + 8u * (no + s);
  }
  __device__ __forceinline__ uint32_t s_full() const { return base + 16 + 16u * nq + 16u * no; }
  __device__ __forceinline__ uint32_t dp_full() const { return s_full() + 8; }
  __device__ __forceinline__ uint32_t s_free() const { return s_full() + 16; }
  __device__ __forceinline__ uint32_t pd_full() const { return s_full() + 24; }
  __device__ __forceinline__ uint32_t acc_done() const { return s_full() + 32; }
  __device__ __forceinline__ uint32_t acc_free() const { return s_full() + 40; }
  __device__ __forceinline__ uint32_t drain() const { return s_full() + 48; }
  __device__ __forceinline__ uint32_t units0() const { return s_full() + 56; }
};

struct KUnit {
  int b, kvh, jb, kt, n;
};

// Units in (batch, K/V head) order, longest first inside a head: K/V block
// j from first to last (a causal K/V block is seen by blocks j..N-1), its
// tiles from first to last.
__device__ __forceinline__ KUnit kv_unit(const BwdParams& p, int u) {
  const int tpb = p.tiles_per_blk;
  const int per_head = p.n_ring * tpb;
  const int bh = u / per_head;
  const int rem = u - bh * per_head;
  KUnit x;
  x.b = bh / p.Hkv;
  x.kvh = bh - x.b * p.Hkv;
  x.jb = rem / tpb;
  x.kt = rem - x.jb * tpb;
  x.n = p.group * (p.causal ? ((tpb - x.kt) + (p.n_ring - 1 - x.jb) * tpb) : p.n_ring * tpb);
  return x;
}

// Query tiles of a K/V unit: blocks i = jb, jb+1, ... (wrapping when not
// causal), within each the heads of the group, within each the tiles (in the
// own block under causal masking only tiles kt.. see this key tile).
struct QWalk {
  int t, i, hh, qt, qt0;
  __device__ __forceinline__ void start(const BwdParams& p, const KUnit& x) {
    t = 0;
    i = x.jb;
    hh = 0;
    qt0 = p.causal ? x.kt : 0;
    qt = qt0;
  }
  __device__ __forceinline__ void next(const BwdParams& p) {
    if (++qt < p.tiles_per_blk) return;
    if (++hh < p.group) {
      qt = qt0;
      return;
    }
    hh = 0;
    ++t;
    i = (i + 1 == p.n_ring) ? 0 : i + 1;
    qt0 = 0;
    qt = 0;
  }
};

template <int D>
__device__ void kv_loader(const BwdParams& p, const KBars& br, const UnitQueue& uq, uint32_t base,
                          float* lse_smem, float* dv_smem, const Ctl& cx) {
  using C = KCfg<D>;
  constexpr int NBOX = D / BOX_COLS;
  const int lane = threadIdx.x & 31;
  uint32_t q_it = 0, units = 0;
  bool kv_pending = false;
  for (int k = 0;; ++k) {
    const int u = uq.take(p.tickets_kv, p.units_kv, k);
    if (u < 0) break;
    const KUnit x = kv_unit(p, u);
    if (units > 0 && !wait_warp(br.kv_empty(), (units - 1) & 1u, cx, SITE_KV_EMPTY)) goto drain;
    {
      const int row = x.b * p.L + x.jb * p.blk_len + x.kt * TM;
      if (elect_one()) {
        mbar_arrive_expect_tx(br.kv_full(), 2 * C::TILE);
#pragma unroll
        for (int bx = 0; bx < NBOX; ++bx) {
          tma_load_3d(base + C::OFF_K + bx * BOX_BYTES, &p.tm_k, br.kv_full(), bx * BOX_COLS, x.kvh, row);
          tma_load_3d(base + C::OFF_V + bx * BOX_BYTES, &p.tm_v, br.kv_full(), bx * BOX_COLS, x.kvh, row);
        }
      }
      __syncwarp();
      kv_pending = true;
    }
    ++units;
    QWalk it;
    it.start(p, x);
    for (int idx = 0; idx < x.n; ++idx, it.next(p)) {
      const int sq = q_it % C::NQ, so = q_it % C::NO;
      const int h = x.kvh * p.group + it.hh;
      const int row = x.b * p.L + it.i * p.blk_len + it.qt * TM;
      // -lse * log2(e) and D of the tile's 128 query rows (rows past the
      // block end: weight 0 through -inf, D = 0), loaded before the waits
      // for the stages so that their latency overlaps them
      const long long vbase = (static_cast<long long>(x.b) * p.Hq + h) * p.L +
                              static_cast<long long>(it.i) * p.blk_len;
      float nlr[TM / 32], dvr[TM / 32];
#pragma unroll
      for (int j = 0; j < TM / 32; ++j) {
        const int qrow = it.qt * TM + lane + 32 * j;
        nlr[j] = -INFINITY;
        dvr[j] = 0.f;
        if (qrow < p.blk_len) {
          nlr[j] = -p.lse[vbase + qrow] * LOG2E;
          dvr[j] = p.dvec[vbase + qrow];
        }
      }
      if (!wait_warp(br.q_empty(sq), ((q_it / C::NQ) & 1u) ^ 1u, cx, SITE_QD_EMPTY)) goto drain;
      if (elect_one()) {
        mbar_arrive_expect_tx(br.q_full(sq), C::TILE);
#pragma unroll
        for (int bx = 0; bx < NBOX; ++bx)
          tma_load_3d(base + C::OFF_Q + sq * C::TILE + bx * BOX_BYTES, &p.tm_q, br.q_full(sq),
                      bx * BOX_COLS, h, row);
      }
#pragma unroll
      for (int j = 0; j < TM / 32; ++j) lse_smem[sq * TM + lane + 32 * j] = nlr[j];
      mbar_arrive(br.q_full(sq));
      if (!wait_warp(br.do_empty(so), ((q_it / C::NO) & 1u) ^ 1u, cx, SITE_QD_EMPTY)) goto drain;
      if (elect_one()) {
        mbar_arrive_expect_tx(br.do_full(so), C::TILE);
#pragma unroll
        for (int bx = 0; bx < NBOX; ++bx)
          tma_load_3d(base + C::OFF_DO + so * C::TILE + bx * BOX_BYTES, &p.tm_do, br.do_full(so),
                      bx * BOX_COLS, h, row);
      }
#pragma unroll
      for (int j = 0; j < TM / 32; ++j) dv_smem[so * TM + lane + 32 * j] = dvr[j];
      mbar_arrive(br.do_full(so));
      ++q_it;
    }
  }
  return;
drain:
  if (lane == 0) {
    // let the copies already issued land before the CTA's shared memory goes
    const uint32_t nq = q_it < static_cast<uint32_t>(C::NQ) ? q_it : C::NQ;
    for (uint32_t i = 0; i < nq; ++i) {
      const uint32_t it = q_it - 1 - i;
      drain_wait(br.q_full(it % C::NQ), (it / C::NQ) & 1u, 200000000ull);
    }
    const uint32_t no = q_it < static_cast<uint32_t>(C::NO) ? q_it : C::NO;
    for (uint32_t i = 0; i < no; ++i) {
      const uint32_t it = q_it - 1 - i;
      drain_wait(br.do_full(it % C::NO), (it / C::NO) & 1u, 200000000ull);
    }
    if (kv_pending) drain_wait(br.kv_full(), (units - 1) & 1u, 200000000ull);
  }
  __syncwarp();
}

template <int D>
__device__ void kv_mma(const BwdParams& p, const KBars& br, const UnitQueue& uq, uint32_t base,
                       uint32_t tmem, const Ctl& cx) {
  using C = KCfg<D>;
  constexpr uint32_t IDESC_S = idesc_bf16_f32(TM, TM, false);
  constexpr uint32_t IDESC_ACC = idesc_bf16_f32(TM, D, true);
  const uint64_t dk0 = smem_desc_sw128(base + C::OFF_K, 16, 1024);
  const uint64_t dv0 = smem_desc_sw128(base + C::OFF_V, 16, 1024);
  const uint64_t dq0 = smem_desc_sw128(base + C::OFF_Q, 16, 1024);
  const uint64_t ddo0 = smem_desc_sw128(base + C::OFF_DO, 16, 1024);
  const uint64_t dqmn0 = smem_desc_sw128(base + C::OFF_Q, BOX_BYTES, 1024);
  const uint64_t ddomn0 = smem_desc_sw128(base + C::OFF_DO, BOX_BYTES, 1024);
  const uint32_t k_lo = static_cast<uint32_t>(dk0), v_lo = static_cast<uint32_t>(dv0);
  const uint32_t q_lo = static_cast<uint32_t>(dq0), do_lo = static_cast<uint32_t>(ddo0);
  const uint32_t qmn_lo = static_cast<uint32_t>(dqmn0), domn_lo = static_cast<uint32_t>(ddomn0);
  const uint32_t hi = static_cast<uint32_t>(dk0 >> 32), mn_hi = static_cast<uint32_t>(dqmn0 >> 32);
  const uint32_t t_s = tmem, t_dp = tmem + 128, t_dv = tmem + 256, t_dk = tmem + 256 + D;
  uint32_t q_it = 0, units = 0, step = 0;
  // S^T = K Q^T (Q stage sq) and dP^T = V dO^T (dO stage so), all K-major
  auto issue_s = [&](int sq) { mma_kmajor<D>(t_s, k_lo, q_lo + ((sq * C::TILE) >> 4), hi, IDESC_S); };
  auto issue_dp = [&](int so) {
    mma_kmajor<D>(t_dp, v_lo, do_lo + ((so * C::TILE) >> 4), hi, IDESC_S);
  };
  for (int k = 0;; ++k) {
    int u;
    if (!uq.read(k, cx, SITE_UNIT, u)) goto drain;
    if (u < 0) break;
    const KUnit x = kv_unit(p, u);
    const int n = x.n;
    if (!wait_warp(br.kv_full(), units & 1u, cx, SITE_KV_FULL)) goto drain;
    {
      const int sq = q_it % C::NQ, so = q_it % C::NO;
      if (!wait_warp(br.q_full(sq), (q_it / C::NQ) & 1u, cx, SITE_QD_FULL)) goto drain;
      tc_fence_after();
      issue_s(sq);
      commit(br.s_full());
      if (!wait_warp(br.do_full(so), (q_it / C::NO) & 1u, cx, SITE_QD_FULL)) goto drain;
      tc_fence_after();
      issue_dp(so);
      commit(br.dp_full());
    }
    for (int idx = 0; idx < n; ++idx) {
      const bool more = idx + 1 < n;
      const int sq = q_it % C::NQ, so = q_it % C::NO;
      const int sq1 = (q_it + 1) % C::NQ, so1 = (q_it + 1) % C::NO;
      if (more) {
        // S^T of the next query tile as soon as the softmax has read this
        // one: P^T and dS^T go to the dP^T columns, so the S^T columns are
        // free from then on and S^T(i+1) overlaps the exponentials of step i
        if (!wait_warp(br.s_free(), step & 1u, cx, SITE_S_FREE)) goto drain;
        if (!wait_warp(br.q_full(sq1), ((q_it + 1) / C::NQ) & 1u, cx, SITE_QD_FULL)) goto drain;
        tc_fence_after();
        issue_s(sq1);
        commit(br.s_full());
      }
      if (!wait_warp(br.pd_full(), step & 1u, cx, SITE_DS_FULL)) goto drain;
      if (idx == 0 && units > 0 &&
          !wait_warp(br.acc_free(), (units - 1) & 1u, cx, SITE_ACC_FREE))
        goto drain;
      tc_fence_after();
      // dV += P^T dO (dO MN-major), P^T pairs at dP^T columns 0-31 / 64-95
      mma_tmem_a_split(t_dv, t_dp, domn_lo + ((so * C::TILE) >> 4), mn_hi, IDESC_ACC,
                       idx > 0 ? 1u : 0u);
      commit(br.do_empty(so));
      // dK += dS^T Q (Q MN-major), dS^T pairs at dP^T columns 32-63 / 96-127
      mma_tmem_a_split(t_dk, t_dp + 32, qmn_lo + ((sq * C::TILE) >> 4), mn_hi, IDESC_ACC,
                       idx > 0 ? 1u : 0u);
      commit(br.q_empty(sq));
      if (more) {
        // dP^T of the next tile overwrites P^T and dS^T after dV and dK have
        // read them (in-order tensor pipe)
        if (!wait_warp(br.do_full(so1), ((q_it + 1) / C::NO) & 1u, cx, SITE_QD_FULL)) goto drain;
        tc_fence_after();
        issue_dp(so1);
        commit(br.dp_full());
      }
      ++step;
      ++q_it;
    }
    commit(br.acc_done());
    commit(br.kv_empty());
    ++units;
  }
  return;
drain:
  commit(br.drain());
  if ((threadIdx.x & 31) == 0) drain_wait(br.drain(), 0u, 200000000ull);
  __syncwarp();
}

template <int D>
__device__ void kv_softmax(const BwdParams& p, const KBars& br, const UnitQueue& uq, uint32_t tmem,
                           const float* lse_smem, const float* dv_smem, int wg, const Ctl& cx) {
  using C = KCfg<D>;
  constexpr int D2 = D / 2;                        // dK, dV columns of this warpgroup
  const int t = threadIdx.x & 127;                 // key row inside the tile
  const int quarter = (threadIdx.x >> 5) & 3;
  const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
  // this warpgroup's queries: columns [64 wg, 64 wg + 64) of S^T and dP^T
  const uint32_t t_s = tmem + lane_off + HALF * wg, t_dp = tmem + lane_off + 128 + HALF * wg;
  const uint32_t t_dv = tmem + lane_off + 256 + D2 * wg, t_dk = tmem + lane_off + 256 + D + D2 * wg;
  const int col0 = HALF * wg;
  const uint64_t c2x2 = f2_pack(p.scale_log2, p.scale_log2);
  uint32_t units = 0, step = 0, q_it = 0;
  for (int k = 0;; ++k) {
    int u;
    if (!uq.read(k, cx, SITE_UNIT, u)) return;
    if (u < 0) break;
    const KUnit x = kv_unit(p, u);
    QWalk it;
    it.start(p, x);
    for (int idx = 0; idx < x.n; ++idx, it.next(p)) {
      const int sq = q_it % C::NQ, so = q_it % C::NO;
      // the diagonal tile of the own block: query column j sees key row t
      // only when j >= t (j > t under the strict mask)
      const bool diag = p.causal && it.i == x.jb && it.qt == x.kt;
      const int first = t + p.diag_shift - col0;   // first allowed local column
      if (!wait_warp(br.s_full(), step & 1u, cx, SITE_S_FULL)) return;
      // the loader's -lse of this Q stage is visible once its phase completed
      // (it completed before S^T was issued)
      if (!wait_warp(br.q_full(sq), (q_it / C::NQ) & 1u, cx, SITE_QD_FULL)) return;
      tc_fence_after();
      const float* nl = lse_smem + sq * TM + col0;
      const float* dvv = dv_smem + so * TM + col0;
      uint32_t sr[64];
      tmem_ld32(t_s, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(t_s + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_wait_ld();
      // S^T is in registers: its columns may take the next tile's S^T
      tc_fence_before();
      mbar_arrive(br.s_free());
      uint32_t pk[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float2 l2 = reinterpret_cast<const float2*>(nl)[j];
        const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(sr[2 * j]), __uint_as_float(sr[2 * j + 1])),
                                   c2x2, f2_pack(l2.x, l2.y));
        float p0, p1;
        f2_unpack(x2, p0, p1);
        p0 = ex2_approx(p0);
        p1 = ex2_approx(p1);
        if (diag) {
          p0 = (2 * j < first) ? 0.f : p0;
          p1 = (2 * j + 1 < first) ? 0.f : p1;
        }
        pk[j] = pack_bf16x2(p0, p1);
      }
      if (!wait_warp(br.dp_full(), step & 1u, cx, SITE_DP_FULL)) return;
      // D of this dO stage (its phase completed before dP^T was issued)
      if (!wait_warp(br.do_full(so), (q_it / C::NO) & 1u, cx, SITE_QD_FULL)) return;
      tc_fence_after();
      {
        // this warpgroup's 64 dP^T columns are read whole, then P^T (pairs,
        // columns 0-31) and dS^T (pairs, columns 32-63) replace them
        uint32_t dp[2][32];
        tmem_ld32(t_dp, dp[0]);
        tmem_ld32(t_dp + 32, dp[1]);
        tmem_wait_ld();
        uint32_t ds[32];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc)
          ds_chunk<true>(*reinterpret_cast<const uint32_t(*)[16]>(&pk[16 * cc]), dp[cc],
                         dvv + 32 * cc, 0.f, *reinterpret_cast<uint32_t(*)[16]>(&ds[16 * cc]));
        tmem_st32(t_dp, pk);
        tmem_st32(t_dp + 32, ds);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(br.pd_full());
      ++step;
      ++q_it;
    }
    // epilogue: dV and dK = scale * (dS^T Q) of this key tile, half the columns
    if (!wait_warp(br.acc_done(), units & 1u, cx, SITE_ACC_DONE)) return;
    tc_fence_after();
    const int krow = x.kt * TM + t;
    const bool valid = krow < p.blk_len;
    const long long off =
        ((static_cast<long long>(x.b) * p.L + static_cast<long long>(x.jb) * p.blk_len + krow) * p.Hkv +
         x.kvh) * D + D2 * wg;
    if (p.dk_acc != nullptr) {
      fold_acc_row<D2>(t_dv, 1.f, p.dv_acc + off, p.fold_kv, nullptr, valid);
      fold_acc_row<D2>(t_dk, p.scale, p.dk_acc + off, p.fold_kv, nullptr, valid);
    } else {
      store_acc_row<D2>(t_dv, 1.f, p.dv + off, valid);
      store_acc_row<D2>(t_dk, p.scale, p.dk + off, valid);
    }
    tc_fence_before();
    mbar_arrive(br.acc_free());
    ++units;
  }
}

template <int D>
__global__ void __launch_bounds__(NUM_THREADS, 1) ra_bwd_dkdv_kernel(const __grid_constant__ BwdParams p) {
  using C = KCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  if (base & 1023u) {
    // the layout has no alignment slack (see KCfg); never seen on B200
    if (threadIdx.x == 0)
      atomicCAS(&g_status, 0ull, (static_cast<unsigned long long>(RA_ERR_UNSUPPORTED) << 32) |
                                     (0xFFFFull << 16) | (blockIdx.x & 0xFFFF));
    return;
  }
  float* lse_smem = reinterpret_cast<float*>(smem_raw + C::OFF_LSE);
  float* dv_smem = reinterpret_cast<float*>(smem_raw + C::OFF_DV);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem_raw + C::OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem_raw + C::OFF_MISC + 4);
  const KBars br{base + C::OFF_BAR, C::NQ, C::NO};
  // as in the dQ kernel, the loader runs at most two units ahead of the
  // softmax warpgroups (unit k + 2 waits for the end of unit k's products)
  const UnitQueue uq{br.units0(), base + C::OFF_UNITS};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0 && lane == 0) {
    mbar_init(br.kv_full(), 1);
    mbar_init(br.kv_empty(), 1);
    for (int s = 0; s < C::NQ; ++s) {
      mbar_init(br.q_full(s), 1 + 32);    // TMA transaction arrive + 32 loader lanes
      mbar_init(br.q_empty(s), 1);
    }
    for (int s = 0; s < C::NO; ++s) {
      mbar_init(br.do_full(s), 1 + 32);
      mbar_init(br.do_empty(s), 1);
    }
    mbar_init(br.s_full(), 1);
    mbar_init(br.dp_full(), 1);
    mbar_init(br.s_free(), SOFTMAX_THREADS);
    mbar_init(br.pd_full(), SOFTMAX_THREADS);
    mbar_init(br.acc_done(), 1);
    mbar_init(br.acc_free(), SOFTMAX_THREADS);
    mbar_init(br.drain(), 1);
    uq.init();
    *abort_flag = 0u;
    fence_mbarrier_init();
  }
  if (warp == WARP_LOAD && lane == 0) {
    prefetch_tensormap(&p.tm_q);
    prefetch_tensormap(&p.tm_do);
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
  const Ctl cx{abort_flag, p.wait_limit_ns, &g_status};
  if (warp < 8) {
    kv_softmax<D>(p, br, uq, tmem, lse_smem, dv_smem, warp >> 2, cx);
  } else if (warp == WARP_LOAD) {
    kv_loader<D>(p, br, uq, base, lse_smem, dv_smem, cx);
  } else {
    kv_mma<D>(p, br, uq, base, tmem, cx);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
static cudaError_t launch_bwd_d(const BwdParams& prm, int num_sms, int max_ctas,
                                cudaStream_t stream) {
  static int configured_dev[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured_dev[dev]) {
    e = cudaFuncSetAttribute(ra_bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             QCfg<D>::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(ra_bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             KCfg<D>::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    configured_dev[dev] = 1;
  }
  auto grid_for = [&](int units) {
    int g = num_sms;
    if (max_ctas > 0 && max_ctas < g) g = max_ctas;
    return units < g ? units : g;
  };
  // each launch takes its units from its own work-queue counter
  BwdParams lp = prm;
  if (prm.parts & 1) {
    e = next_ticket_counter(stream, &lp.tickets_dq);
    if (e != cudaSuccess) return e;
    ra_bwd_dq_kernel<D><<<grid_for(prm.units_dq), NUM_THREADS, QCfg<D>::SMEM_BYTES, stream>>>(lp);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (prm.parts & 2) {
    e = next_ticket_counter(stream, &lp.tickets_kv);
    if (e != cudaSuccess) return e;
    ra_bwd_dkdv_kernel<D><<<grid_for(prm.units_kv), NUM_THREADS, KCfg<D>::SMEM_BYTES, stream>>>(lp);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace bwd

cudaError_t launch_bwd(const BwdParams& prm, int d, int num_sms, int max_ctas,
                       cudaStream_t stream) {
  if (d == 128) return bwd::launch_bwd_d<128>(prm, num_sms, max_ctas, stream);
  return bwd::launch_bwd_d<64>(prm, num_sms, max_ctas, stream);
}

// Fixed device scratch for ring_attn_bwd_noalloc: one fp32 D value per query
// row and head, for problems with B * Hq * L <= kNoAllocScratchRows.  It is
// part of the module image (no allocation call creates it); every call
// overwrites the entries it reads, so nothing in it has to start at zero.
__device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchRows];

cudaError_t noalloc_scratch(void** ptr, cudaStream_t stream) {
  return symbol_address(reinterpret_cast<const void*>(&g_noalloc_scratch), ptr, stream);
}

cudaError_t read_and_clear_bwd_status(unsigned long long* out) {
  unsigned long long v = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, bwd::g_status, sizeof(v));
  if (e != cudaSuccess) return e;
  if (v != 0) {
    e = cudaMemcpyToSymbol(bwd::g_status, &zero, sizeof(zero));
    if (e != cudaSuccess) return e;
  }
  *out = v;
  return cudaSuccess;
}

}  // namespace ra
