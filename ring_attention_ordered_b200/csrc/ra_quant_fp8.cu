// Block quantisation to E4M3 for the FP8 forward (sm_100a).
//
// The FlashAttention article (developer.aliyun page, section 二,
// FlashAttention-3 改进) keeps FP8 precision loss down by quantising in
// blocks.  Here a block is the 128-row tile of one (batch, head): its scale is
// amax / 448 in float32 (1 for an all-zero tile), and each element becomes
// E4M3(x / scale), the quotient rounded to float32 (IEEE division) and then to
// E4M3 with ties to even, saturating at +-448.  A ragged last tile holds the
// remaining rows.
//
// One CTA per (tile, head, batch), 256 threads: a first pass of 16-byte loads
// reduces |x| to the tile's maximum (packed bf16 maxima), a second pass
// reads the tile again (an L2 hit) and writes the codes (8 bytes per store)
// and the scale.  The algorithmic traffic is 2 bytes read and 1 byte written
// per element; the instruction count per element is kept low (chunk
// indices from compile-time shifts for d = 64, 128 and 256, packed f32x2
// arithmetic for the quotient) so that issue does not bound the kernel.
//
// The quotient x / s is formed without a division per element (Markstein's
// method for correctly rounded division): once per tile, s is scaled by a
// power of two c into s1 = s c in [1, 2) and r1 = 1/s1 is rounded to
// nearest; per element x1 = x c (exact), q0 = x1 r1 and one residual
// correction q = q0 + (x1 - q0 s1) r1 with fused multiply-adds.  The scaling
// keeps the residual clear of underflow.  For the operands this kernel sees
// -- x a bf16 value and s = amax / 448 rounded to float32 with amax a bf16
// value -- the E4M3 code of q equals that of the IEEE quotient: checked
// exhaustively on a B200 for every finite bf16 x and every positive finite
// bf16 amax (2^31 pairs).  Tiles whose s is not a normal float (amax below
// 448 x 2^-126) take the IEEE division.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx_sm100.cuh"
#include "ra_internal.h"

namespace ra {
namespace {

constexpr int QT = 256;             // threads per CTA
constexpr int ROWS = 128;           // rows per tile
constexpr int MAX_CHUNKS = 16;      // 16-byte chunks per thread: 128 rows x 256 cols / 8 / 256

__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Elementwise max of |x| over the 8 bf16 values of a chunk, on packed pairs.
__device__ __forceinline__ __nv_bfloat162 absmax8(uint4 v, __nv_bfloat162 m) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) m = __hmax2(m, __habs2(h[i]));
  return m;
}

// x / s as described in the file comment: c = 2^-e for s = 2^e (1 + f),
// s1 = s c, r1 = 1/s1 rounded to nearest; pairs hold the same value twice.
struct Divisor {
  float s;
  uint64_t c2, s1n2, r12;
  bool fast;
};

__device__ __forceinline__ Divisor make_divisor(float s) {
  Divisor d;
  d.s = s;
  d.fast = s >= 1.17549435e-38f;   // normal float
  const uint32_t ef = (__float_as_uint(s) >> 23) & 0xffu;
  const float c = __uint_as_float((254u - ef) << 23);
  const float s1 = s * c;
  const float r1 = __frcp_rn(s1);
  d.c2 = f2_pack(c, c);
  d.s1n2 = f2_pack(-s1, -s1);
  d.r12 = f2_pack(r1, r1);
  return d;
}

// E4M3 codes of two bf16 values (a bf16x2 word) divided by the scale.
__device__ __forceinline__ uint32_t quantize_pair(uint32_t xb, const Divisor& d) {
  const float x0 = __uint_as_float(xb << 16);
  const float x1 = __uint_as_float(xb & 0xffff0000u);
  float q0, q1;
  if (d.fast) {
    const uint64_t xs = f2_mul(f2_pack(x0, x1), d.c2);        // exact: power-of-two scaling
    const uint64_t p = f2_mul(xs, d.r12);
    const uint64_t q = f2_fma(f2_fma(p, d.s1n2, xs), d.r12, p);
    f2_unpack(q, q0, q1);
    // the sign of x: a quotient too small for E4M3 must round to the zero
    // of x's sign, which the correction step can lose when it returns zero
    q0 = copysignf(q0, x0);
    q1 = copysignf(q1, x1);
  } else {
    q0 = __fdiv_rn(x0, d.s);
    q1 = __fdiv_rn(x1, d.s);
  }
  return e4m3x2(q0, q1);
}

// CPR: 16-byte chunks per row (d / 8) when known at compile time, else 0.
template <int CPR>
__global__ void __launch_bounds__(QT) ra_quant_fp8_kernel(const __nv_bfloat16* __restrict__ x,
                                                          uint8_t* __restrict__ codes,
                                                          float* __restrict__ scales, long long L,
                                                          int H, int d, int T) {
  __shared__ float red[QT / 32];
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const long long r0 = static_cast<long long>(t) * ROWS;
  const int rows = static_cast<int>(min(static_cast<long long>(ROWS), L - r0));
  const int cpr = CPR ? CPR : d / 8;             // 16-byte chunks per row
  const int n = rows * cpr;
  const long long row_stride = static_cast<long long>(H) * d;
  const long long base = (static_cast<long long>(b) * L + r0) * row_stride + static_cast<long long>(h) * d;
  constexpr int NCH = CPR ? (ROWS * CPR + QT - 1) / QT : MAX_CHUNKS;

  // pass 1: the tile's maximum magnitude (loads only, all in flight at once)
  __nv_bfloat162 m2 = __float2bfloat162_rn(0.f);
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    const int c = threadIdx.x + i * QT;
    if (c < n) {
      const int r = c / cpr, cc = c % cpr;
      m2 = absmax8(__ldg(reinterpret_cast<const uint4*>(x + base + r * row_stride) + cc), m2);
    }
  }
  float m = fmaxf(__low2float(m2), __high2float(m2));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  float amax = red[0];
#pragma unroll
  for (int i = 1; i < QT / 32; ++i) amax = fmaxf(amax, red[i]);
  const float s = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  const Divisor dv = make_divisor(s);
  if (threadIdx.x == 0) scales[(static_cast<long long>(b) * H + h) * T + t] = s;

  // pass 2: read the tile again (from L2: it was read a moment ago) and
  // write the codes.
#pragma unroll 4
  for (int i = 0; i < NCH; ++i) {
    const int c = threadIdx.x + i * QT;
    if (c < n) {
      const int r = c / cpr, cc = c % cpr;
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(x + base + r * row_stride) + cc);
      uint2 out;
      out.x = quantize_pair(v.x, dv) | (quantize_pair(v.y, dv) << 16);
      out.y = quantize_pair(v.z, dv) | (quantize_pair(v.w, dv) << 16);
      *(reinterpret_cast<uint2*>(codes + base + r * row_stride) + cc) = out;
    }
  }
}

}  // namespace

cudaError_t launch_quantize_fp8(const __nv_bfloat16* x, uint8_t* codes, float* scales, int B,
                                long long L, int H, int d, cudaStream_t stream) {
  const long long T = (L + ROWS - 1) / ROWS;
  if (T > 0x7fffffffll || H > 65535 || B > 65535) return cudaErrorInvalidValue;
  if (d % 8 != 0 || d < 8 || d > 256) return cudaErrorInvalidValue;
  dim3 grid(static_cast<unsigned>(T), static_cast<unsigned>(H), static_cast<unsigned>(B));
  const int Ti = static_cast<int>(T);
  if (d == 128)
    ra_quant_fp8_kernel<16><<<grid, QT, 0, stream>>>(x, codes, scales, L, H, d, Ti);
  else if (d == 64)
    ra_quant_fp8_kernel<8><<<grid, QT, 0, stream>>>(x, codes, scales, L, H, d, Ti);
  else if (d == 256)
    ra_quant_fp8_kernel<32><<<grid, QT, 0, stream>>>(x, codes, scales, L, H, d, Ti);
  else
    ra_quant_fp8_kernel<0><<<grid, QT, 0, stream>>>(x, codes, scales, L, H, d, Ti);
  return cudaGetLastError();
}

}  // namespace ra
