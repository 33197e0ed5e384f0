// FP8 (E4M3) forward of ring-ordered blockwise attention for sm_100a, d = 128.
//
// What it computes: the ring-ordered forward of the bf16 kernel (the same
// work units, ring order (i - t) mod n_ring, causal skipping and diagonal
// masking; "Ring Attention 环注意力", L3 definition, L4 §4.2 and §4.5) on
// block-quantised inputs -- the FP8 forward of the FlashAttention article
// (developer.aliyun page, section 二, FlashAttention-3 改进): both GEMMs run
// on the FP8 tensor cores, and q, k and v carry one float32 scale per 128-row
// tile of each (batch, head).  The result approximates exact attention of the
// dequantised tensors code * scale; the only coarse rounding is that of the
// probabilities to E4M3 before the P V product.
//
// How (differences from the bf16 kernel):
//   * S = Q8 K8^T by tcgen05.mma kind::f8f6f4 (E4M3 x E4M3, f32 in TMEM),
//     4 MMAs of K = 32; the softmax multiplies S by
//     scale * log2(e) * sq(query tile) * sk(key tile);
//   * P' = 2^(x - m) * f_j with f_j = sv_j / R (R = the largest V scale of the
//     batch's K/V head) is rounded to E4M3 and stored over S, four keys per
//     TMEM column, so O accumulates P' V8 in units of R and tiles with
//     different V scales add up exactly; the factor f_j rides in the
//     exponent's bias, at no cost.  The row sum takes the unrounded 2^(x - m);
//     the epilogue multiplies O by R / l;
//   * tiles are 16 KB: one TMA box (128 rows x 128 bytes, 128-byte swizzle)
//     per tile and 8 K/V stages; V is read as an MN-major B operand.
//   The loader and MMA roles, the work queue and the barriers are the bf16
//   kernel's (ra_fwd_roles.cuh, with this kernel's tile geometry); the
//   softmax keeps a lazy rescale (threshold 2^8, so P' <= 256 stays below
//   E4M3's 448).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx_sm100.cuh"
#include "ra_fwd_roles.cuh"
#include "ra_internal.h"
#include "ra_schedule.cuh"
#include "ra_sync.cuh"
#include "ring_attn.h"

namespace ra {
namespace fp8 {

constexpr int BM = FWD_BM;
constexpr int BN = FWD_BN;
constexpr int D = 128;
constexpr int TILE_BYTES = 128 * 128;   // 128 rows x 128 E4M3 values
constexpr int NUM_THREADS = 384;
constexpr int WARP_LOAD = 8;
constexpr int WARP_MMA = 9;
constexpr int LAUNCH_REGS = 168;
constexpr int SOFTMAX_REGS = 224;
constexpr int CONTROL_REGS = 56;
static_assert(2 * 128 * SOFTMAX_REGS + 128 * CONTROL_REGS <= NUM_THREADS * LAUNCH_REGS,
              "register split exceeds the launch allocation");
constexpr float RESCALE_LOG2 = 8.0f;
constexpr float LN2 = 0.69314718055994530942f;

constexpr int NS = 8;                         // K/V stages
constexpr int OFF_Q = 0;
constexpr int OFF_KV = 2 * TILE_BYTES;
constexpr int OFF_BAR = OFF_KV + NS * TILE_BYTES;
// barriers (ra_fwd_roles.cuh), then tmem holder + abort flag, then the unit
// queue
constexpr int OFF_MISC = OFF_BAR + fwd_num_bars(NS) * 8;
constexpr int OFF_UNITS = OFF_MISC + 16;
constexpr int SMEM_BYTES = OFF_UNITS + UQ * 4 + 1024;   // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

__device__ unsigned long long g_status = 0ull;

// ------------------------------------------------------------------ MMA
// S = Q8 K8^T: 4 MMAs of K = 32 (32 bytes apart inside the 128-byte swizzle
// row; descriptor offsets in 16-byte units).
__device__ __forceinline__ void mma_qk(uint32_t d, uint32_t a, uint32_t b, uint32_t hi,
                                       uint32_t idesc) {
  if (elect_one()) mma_ss_f8<0, 0>(d, a, hi, b, hi, idesc, 0u);
  if (elect_one()) mma_ss_f8<2, 2>(d, a, hi, b, hi, idesc, 1u);
  if (elect_one()) mma_ss_f8<4, 4>(d, a, hi, b, hi, idesc, 1u);
  if (elect_one()) mma_ss_f8<6, 6>(d, a, hi, b, hi, idesc, 1u);
}

// O (+)= P' V8 over one half of the 128 keys: 2 MMAs of K = 32.  P' holds
// four keys per TMEM column (32 keys = 8 columns); V's 32 keys are 32 rows
// of 128 bytes (4096 bytes = 256 descriptor units).
template <int HALF>
__device__ __forceinline__ void mma_pv_half(uint32_t d, uint32_t p_tmem, uint32_t b, uint32_t hi,
                                            uint32_t idesc, uint32_t acc) {
  constexpr uint32_t C0 = 16 * HALF, B0 = 512 * HALF;
  if (elect_one()) mma_ts_f8<C0 + 0, B0 + 0>(d, p_tmem, b, hi, idesc, HALF ? 1u : acc);
  if (elect_one()) mma_ts_f8<C0 + 8, B0 + 256>(d, p_tmem, b, hi, idesc, 1u);
}

// Geometry of the FP8 kernel for the shared loader and MMA roles: a tile is
// one TMA box of 128 rows x 128 bytes (one 128-byte swizzle row per row);
// tcgen05.mma kind::f8f6f4 with K = 32.
struct Fp8Geom {
  static constexpr int Q_BYTES = TILE_BYTES;
  static constexpr int KV_BYTES = TILE_BYTES;
  static constexpr int NS = fp8::NS;
  static constexpr int OFF_Q = fp8::OFF_Q;
  static constexpr int OFF_KV = fp8::OFF_KV;
  static constexpr uint32_t IDESC_QK = idesc_e4m3_f32(BM, BN, false);
  static constexpr uint32_t IDESC_PV = idesc_e4m3_f32(BM, D, true);

  static __device__ __forceinline__ void load_q(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                                int h, int row) {
    tma_load_3d(dst, map, bar, 0, h, row);
  }
  static __device__ __forceinline__ void load_kv(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t bar, int h, int row) {
    tma_load_3d(dst, map, bar, 0, h, row);
  }

  // Descriptor low words (start address in 16-byte units below 2^18 bytes,
  // so added offsets never carry out of the field) and the shared high word.
  // V is MN-major: its 128 E4M3 values per key span exactly one 128-byte
  // swizzle atom along N, so the atom stride (leading byte offset) is never
  // used; it is set to 16 bytes, which keeps even a misread inside the tile.
  uint32_t q_lo, k_lo, v_lo, k_hi, v_hi;
  __device__ explicit Fp8Geom(uint32_t smem_base) {
    const uint64_t dq0 = smem_desc_sw128(smem_base + OFF_Q, 16, 1024);
    const uint64_t dkv0 = smem_desc_sw128(smem_base + OFF_KV, 16, 1024);
    q_lo = static_cast<uint32_t>(dq0);
    k_lo = static_cast<uint32_t>(dkv0);
    v_lo = static_cast<uint32_t>(dkv0);
    k_hi = static_cast<uint32_t>(dkv0 >> 32);
    v_hi = static_cast<uint32_t>(dkv0 >> 32);
  }
  __device__ __forceinline__ void issue_qk(uint32_t d, int w, int stage) const {
    mma_qk(d, q_lo + ((w * TILE_BYTES) >> 4), k_lo + ((stage * TILE_BYTES) >> 4), k_hi, IDESC_QK);
  }
  template <int HALF>
  __device__ __forceinline__ void issue_pv_half(uint32_t d, uint32_t p_tmem, int stage,
                                                uint32_t acc) const {
    mma_pv_half<HALF>(d, p_tmem, v_lo + ((stage * TILE_BYTES) >> 4), v_hi, IDESC_PV, acc);
  }
};

// ------------------------------------------------------------------ softmax
// One score row (128 columns in sr): P' = 2^(s * c2 + bias) rounded to E4M3
// and written to TMEM columns [0, 32) at tS, four keys per column, the first
// 64 keys before the arrival on p_half_bar.  Returns the fp32 sum of the
// unrounded P'.  MASKED: columns > lim get exactly zero.  Warp-collective
// (tcgen05.st): all 32 lanes call the same instantiation together.
template <bool MASKED>
__device__ __forceinline__ float exp_row_store(uint32_t (&sr)[128], float c2, float bias, int lim,
                                               uint32_t tS, uint32_t p_half_bar) {
  const uint64_t c2x2 = f2_pack(c2, c2);
  const uint64_t b2 = f2_pack(bias, bias);
  uint64_t acc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i] = f2_pack(0.f, 0.f);
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    uint32_t pk[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int col = 64 * half + 4 * j;
      const uint64_t xa = f2_fma(f2_pack(__uint_as_float(sr[col]), __uint_as_float(sr[col + 1])),
                                 c2x2, b2);
      const uint64_t xb = f2_fma(
          f2_pack(__uint_as_float(sr[col + 2]), __uint_as_float(sr[col + 3])), c2x2, b2);
      float x0, x1, x2, x3;
      f2_unpack(xa, x0, x1);
      f2_unpack(xb, x2, x3);
      float p0 = ex2_approx(x0), p1 = ex2_approx(x1), p2 = ex2_approx(x2), p3 = ex2_approx(x3);
      if (MASKED) {
        p0 = (col > lim) ? 0.f : p0;
        p1 = (col + 1 > lim) ? 0.f : p1;
        p2 = (col + 2 > lim) ? 0.f : p2;
        p3 = (col + 3 > lim) ? 0.f : p3;
      }
      acc[(2 * j) & 3] = f2_add(acc[(2 * j) & 3], f2_pack(p0, p1));
      acc[(2 * j + 1) & 3] = f2_add(acc[(2 * j + 1) & 3], f2_pack(p2, p3));
      pk[j] = pack_e4m3x4(p0, p1, p2, p3);
    }
    tmem_st16(tS + 16 * half, pk);
    if (half == 0) {
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

__device__ void softmax_role(const Fp8FwdParams& p, const FwdBars& br, uint32_t tmem, int w,
                             const Ctl& cx) {
  const int t = threadIdx.x - w * 128;
  const int lane = threadIdx.x & 31;
  const int quarter = (threadIdx.x >> 5) & 3;
  const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t tS = tmem + lane_off + w * 128;  // S (fp32), then P' (E4M3, first 32 columns)
  const uint32_t tO = tmem + lane_off + 256 + w * 128;
  uint32_t s_phase = 0u, units_w = 0u;
  int r_head = -1;          // (batch, K/V head) whose R is cached
  float R = 1.f, log2R = 0.f;

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
    const int qrow = qt * BM + t;
    const int head = x.b * p.Hkv + x.kvh;
    const float* skh = p.sk + static_cast<long long>(head) * p.n_tiles;
    const float* svh = p.sv + static_cast<long long>(head) * p.n_tiles;
    if (head != r_head) {
      // R = the largest V scale of this (batch, K/V head), reduced per warp
      float r = 0.f;
      for (int i = lane; i < p.n_tiles; i += 32) r = fmaxf(r, __ldg(svh + i));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) r = fmaxf(r, __shfl_xor_sync(0xffffffffu, r, o));
      R = r;
      log2R = __log2f(r);
      r_head = head;
    }
    const float c2q =
        p.scale_log2 *
        __ldg(p.sq + (static_cast<long long>(x.b) * p.Hq + h) * p.n_tiles + x.blk * p.tiles_per_blk + qt);
    float m = -INFINITY, l = 0.f;
    KvIter it;
    it.start(p, x);

    for (int idx = 0; idx < x.n_kv; ++idx, it.next(p)) {
      const int kt = it.jb * p.tiles_per_blk + it.kl;
      const float skj = __ldg(skh + kt);
      const float svj = __ldg(svh + kt);
      int lim = BN - 1;
      if (p.causal && it.jb == x.blk) lim = min(lim, qrow - it.kl * BN);
      const bool masked = __any_sync(0xffffffffu, lim < BN - 1);

      bool ok = wait_bar(br.s_full(w), s_phase, cx, SITE_S_FULL);
      if (!__all_sync(0xffffffffu, ok)) return;
      s_phase ^= 1u;
      tc_fence_after();

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
      // log2-domain multiplier of this tile pair (>= 0, so the max commutes)
      const float c2 = c2q * skj;
      const float m_tile = (rmax == -INFINITY) ? -INFINITY : rmax * c2;
      const bool need = m_tile > m + RESCALE_LOG2;
      float alpha = 1.f;
      if (__any_sync(0xffffffffu, need)) {
        const float m_new = need ? m_tile : m;
        alpha = (m_new == m) ? 1.f : ex2_approx(m - m_new);
        if (idx > 0) {
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
      // log2 of this tile's V-scale fraction f_j = sv_j / R (<= 0), folded
      // into the exponent; the row sum is brought back by 2^-lf
      const float lf = __log2f(svj) - log2R;
      const float rsum = masked ? exp_row_store<true>(sr, c2, lf - m, lim, tS, br.p_half(w))
                                : exp_row_store<false>(sr, c2, lf - m, lim, tS, br.p_half(w));
      l = l * alpha + rsum * ex2_approx(-lf);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(br.p_full(w));
    }

    // epilogue: O * R / l in bf16, lse = (m + log2 l) ln 2
    {
      bool ok = wait_bar(br.o_done(w), units_w & 1u, cx, SITE_O_DONE);
      if (!__all_sync(0xffffffffu, ok)) return;
      tc_fence_after();
      const long long pos = static_cast<long long>(x.blk) * p.blk_len + qrow;
      const float f_out = R / l;
      __nv_bfloat16* dst = p.out + ((static_cast<long long>(x.b) * p.L + pos) * p.Hq + h) * D;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tmem_ld32(tO + cc * 32, o);
        tmem_wait_ld();
        uint32_t pkd[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          pkd[j] = pack_bf16x2(__uint_as_float(o[2 * j]) * f_out, __uint_as_float(o[2 * j + 1]) * f_out);
        uint4* d4 = reinterpret_cast<uint4*>(dst + cc * 32);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          d4[j] = make_uint4(pkd[4 * j], pkd[4 * j + 1], pkd[4 * j + 2], pkd[4 * j + 3]);
      }
      tc_fence_before();
      mbar_arrive(br.o_free(w));
      p.lse[(static_cast<long long>(x.b) * p.Hq + h) * p.L + pos] = (m + log2f(l)) * LN2;
      ++units_w;
    }
  }
}

// ------------------------------------------------------------------ kernel
__global__ void __launch_bounds__(NUM_THREADS, 1)
    ra_fwd_fp8_kernel(const __grid_constant__ Fp8FwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);

  FwdBars br;
  br.layout(base + OFF_BAR, NS, base + OFF_UNITS);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(base_ptr + OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(base_ptr + OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    br.init(NS);
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
  const Ctl cx{abort_flag, p.wait_limit_ns, &g_status};

  if (warp < 8) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" :: "n"(SOFTMAX_REGS));
    softmax_role(p, br, tmem, warp >> 2, cx);
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" :: "n"(CONTROL_REGS));
    if (warp == WARP_LOAD) {
      fwd_loader_role<Fp8Geom>(p, br, base, cx);
    } else if (warp == WARP_MMA) {
      fwd_mma_role<Fp8Geom>(p, br, base, tmem, cx);
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

}  // namespace fp8

// ------------------------------------------------------------------ host
cudaError_t launch_fwd_fp8(const Fp8FwdParams& prm, int grid, cudaStream_t stream) {
  static int configured_dev[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured_dev[dev]) {
    // the setmaxnreg split needs exactly LAUNCH_REGS registers per thread
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, fp8::ra_fwd_fp8_kernel);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != fp8::LAUNCH_REGS) return cudaErrorInvalidKernelImage;
    e = cudaFuncSetAttribute(fp8::ra_fwd_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             fp8::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    configured_dev[dev] = 1;
  }
  fp8::ra_fwd_fp8_kernel<<<grid, fp8::NUM_THREADS, fp8::SMEM_BYTES, stream>>>(prm);
  return cudaGetLastError();
}

cudaError_t read_and_clear_fp8_status(unsigned long long* out) {
  unsigned long long v = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, fp8::g_status, sizeof(v));
  if (e != cudaSuccess) return e;
  if (v != 0) {
    e = cudaMemcpyToSymbol(fp8::g_status, &zero, sizeof(zero));
    if (e != cudaSuccess) return e;
  }
  *out = v;
  return cudaSuccess;
}

}  // namespace ra
