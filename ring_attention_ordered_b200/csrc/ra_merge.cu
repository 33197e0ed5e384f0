// Log-sum-exp merge of two partial attention results (sm_100a).
//
// The pages fold each ring step's blockwise result into the running output
// ("Ring Attention 环注意力", L4 §4.2 step 2) and keep only the logsumexp
// statistic (FlashAttention article, FlashAttention-2 改进).  For two partials
// over disjoint key sets:
//   M = max(lse_a, lse_b), w = exp(lse - M),
//   lse = M + ln(w_a + w_b), o = (w_a o_a + w_b o_b) / (w_a + w_b).
//
// The kernel is a single streaming pass over HBM (3 * (4d + 4) bytes per
// row): each warp handles four rows at a time, lanes stride over the row in
// 16-byte vectors, the two lse values of a row are read by every lane before
// lane r writes lse_out of row r, so in-place use (out == a or out == b) is
// safe.  Products and sums are rounded explicitly (no FMA contraction) so that
// swapping a and b gives a bitwise identical result.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "ra_internal.h"
#include "ra_merge_math.cuh"

namespace ra {

constexpr int MERGE_ROWS = 4;
constexpr int MERGE_THREADS = 256;

__global__ void __launch_bounds__(MERGE_THREADS) ra_merge_kernel(
    const float* o_a, const float* lse_a, const float* o_b, const float* lse_b, float* o_out,
    float* lse_out, long long rows, int d) {
  const int lane = threadIdx.x & 31;
  const long long warp = (static_cast<long long>(blockIdx.x) * MERGE_THREADS + threadIdx.x) >> 5;
  const long long nwarps = (static_cast<long long>(gridDim.x) * MERGE_THREADS) >> 5;
  const int d4 = d >> 2;
  for (long long r0 = warp * MERGE_ROWS; r0 < rows; r0 += nwarps * MERGE_ROWS) {
    MergeW w[MERGE_ROWS];
#pragma unroll
    for (int r = 0; r < MERGE_ROWS; ++r) {
      const long long row = r0 + r;
      const float la = row < rows ? lse_a[row] : -INFINITY;
      const float lb = row < rows ? lse_b[row] : -INFINITY;
      w[r] = merge_weights(la, lb);
    }
    for (int c4 = lane; c4 < d4; c4 += 32) {
      float4 va[MERGE_ROWS], vb[MERGE_ROWS];
#pragma unroll
      for (int r = 0; r < MERGE_ROWS; ++r) {
        const long long row = r0 + r;
        if (row < rows) {
          va[r] = reinterpret_cast<const float4*>(o_a + row * d)[c4];
          vb[r] = reinterpret_cast<const float4*>(o_b + row * d)[c4];
        }
      }
#pragma unroll
      for (int r = 0; r < MERGE_ROWS; ++r) {
        const long long row = r0 + r;
        if (row < rows) {
          float4 o;
          o.x = merge_one(w[r], va[r].x, vb[r].x);
          o.y = merge_one(w[r], va[r].y, vb[r].y);
          o.z = merge_one(w[r], va[r].z, vb[r].z);
          o.w = merge_one(w[r], va[r].w, vb[r].w);
          reinterpret_cast<float4*>(o_out + row * d)[c4] = o;
        }
      }
    }
    __syncwarp();
    if (lane < MERGE_ROWS && r0 + lane < rows) {
      float lv = w[0].lse;
#pragma unroll
      for (int r = 1; r < MERGE_ROWS; ++r)
        if (lane == r) lv = w[r].lse;
      lse_out[r0 + lane] = lv;
    }
  }
}

// fp32 -> bf16, round to nearest even: 8 elements (32 bytes in, 16 out) per
// thread and loop trip, grid-stride.
__global__ void __launch_bounds__(256) ra_round_bf16_kernel(const float4* __restrict__ src,
                                                            uint4* __restrict__ dst, long long n8) {
  for (long long i = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * 256) {
    const float4 a = src[2 * i], b = src[2 * i + 1];
    uint4 o;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(o.x) : "f"(a.y), "f"(a.x));
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(o.y) : "f"(a.w), "f"(a.z));
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(o.z) : "f"(b.y), "f"(b.x));
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(o.w) : "f"(b.w), "f"(b.z));
    dst[i] = o;
  }
}

cudaError_t launch_round_bf16(const float* src, __nv_bfloat16* dst, long long n, int num_sms,
                              cudaStream_t stream) {
  const long long n8 = n / 8;
  long long grid = (n8 + 255) / 256;
  if (grid > static_cast<long long>(num_sms) * 8) grid = static_cast<long long>(num_sms) * 8;
  if (grid < 1) grid = 1;
  ra_round_bf16_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(
      reinterpret_cast<const float4*>(src), reinterpret_cast<uint4*>(dst), n8);
  return cudaGetLastError();
}

cudaError_t launch_merge(const float* o_a, const float* lse_a, const float* o_b,
                         const float* lse_b, float* o_out, float* lse_out, long long rows, int d,
                         int num_sms, cudaStream_t stream) {
  const long long warps_needed = (rows + MERGE_ROWS - 1) / MERGE_ROWS;
  const long long blocks_needed = (warps_needed + (MERGE_THREADS / 32) - 1) / (MERGE_THREADS / 32);
  long long grid = static_cast<long long>(num_sms) * 8;
  if (grid > blocks_needed) grid = blocks_needed;
  if (grid < 1) grid = 1;
  ra_merge_kernel<<<static_cast<unsigned>(grid), MERGE_THREADS, 0, stream>>>(
      o_a, lse_a, o_b, lse_b, o_out, lse_out, rows, d);
  return cudaGetLastError();
}

}  // namespace ra
