// Log-sum-exp merge of two partial attention results over disjoint key sets,
// one row at a time (used by the merge kernel and by the fused fold of the
// per-visit forward kernel, so both give bitwise the same result):
//   M = max(lse_a, lse_b), w = exp(lse - M),
//   lse = M + ln(w_a + w_b), o = (w_a o_a + w_b o_b) / (w_a + w_b).
// A partial with lse = -inf is empty and its o is ignored (even NaN); two
// empty partials give o = 0, lse = -inf; NaN in an lse makes the row NaN.
// Products and sums are rounded explicitly (no FMA contraction), so swapping
// a and b gives a bitwise identical result.
#pragma once

#include <cuda_runtime.h>

#include <cmath>

namespace ra {

struct MergeW {
  float wa, wb, inv, lse;
  int mode;  // 0 normal, 1 both empty, 2 NaN
};

__device__ __forceinline__ MergeW merge_weights(float la, float lb) {
  MergeW w;
  if (isnan(la) || isnan(lb)) {
    w.mode = 2;
    w.wa = w.wb = w.inv = w.lse = __int_as_float(0x7fc00000);
    return w;
  }
  const float mx = fmaxf(la, lb);
  if (mx == -INFINITY) {
    w.mode = 1;
    w.wa = w.wb = 0.f;
    w.inv = 0.f;
    w.lse = -INFINITY;
    return w;
  }
  w.mode = 0;
  w.wa = expf(la - mx);
  w.wb = expf(lb - mx);
  const float den = __fadd_rn(w.wa, w.wb);
  w.inv = __frcp_rn(den);
  w.lse = mx + logf(den);
  return w;
}

__device__ __forceinline__ float merge_one(const MergeW& w, float a, float b) {
  if (w.mode == 1) return 0.f;
  if (w.mode == 2) return w.lse;
  const float ta = (w.wa == 0.f) ? 0.f : __fmul_rn(w.wa, a);
  const float tb = (w.wb == 0.f) ? 0.f : __fmul_rn(w.wb, b);
  return __fmul_rn(__fadd_rn(ta, tb), w.inv);
}

}  // namespace ra
