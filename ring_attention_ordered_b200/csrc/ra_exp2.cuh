// 2^x on the FMA pipe instead of the MUFU ex2 unit (sm_100a), for kernels
// whose exponentials limit a dependency chain: moving part of them to the
// otherwise idle FMA pipe shortens the MUFU-bound stretch.
#pragma once

#include <cstdint>

#include "ptx_sm100.cuh"

namespace ra {

// Minimax (relative error) cubic for 2^f on [-1/2, 1/2], fitted by
// csrc/fit_exp2_poly.py (Remez exchange); max relative error 7.5e-5 with
// float32 Horner evaluation.
constexpr float EXP2_C0 = 9.999280572e-01f;
constexpr float EXP2_C1 = 6.932609677e-01f;
constexpr float EXP2_C2 = 2.426111251e-01f;
constexpr float EXP2_C3 = 5.517166853e-02f;

// 2^x for two values at once on the FMA pipe: x = j + f with j = round(x)
// (adding and subtracting 1.5 * 2^23 rounds to the nearest integer), p(f) by
// the cubic above, then 2^j applied by adding j << 23 to the bits of p(f)
// (the low bits of x + 1.5 * 2^23 hold j in two's complement).  Inputs are
// clamped to >= -125 so the scaled result stays a normal float; anything
// below 2^-125 is negligible next to the row maximum's 2^0.
__device__ __forceinline__ void exp2_poly2(uint64_t x2, float& r0, float& r1) {
  float a, b;
  f2_unpack(x2, a, b);
  x2 = f2_pack(fmaxf(a, -125.f), fmaxf(b, -125.f));
  const uint64_t magic = f2_pack(12582912.f, 12582912.f);
  const uint64_t neg_magic = f2_pack(-12582912.f, -12582912.f);
  const uint64_t t = f2_add(x2, magic);
  const uint64_t j = f2_add(t, neg_magic);
  const uint64_t f = f2_fma(j, f2_pack(-1.f, -1.f), x2);
  uint64_t q = f2_fma(f2_pack(EXP2_C3, EXP2_C3), f, f2_pack(EXP2_C2, EXP2_C2));
  q = f2_fma(q, f, f2_pack(EXP2_C1, EXP2_C1));
  q = f2_fma(q, f, f2_pack(EXP2_C0, EXP2_C0));
  float q0, q1, t0, t1;
  f2_unpack(q, q0, q1);
  f2_unpack(t, t0, t1);
  r0 = __uint_as_float(__float_as_uint(q0) + __float_as_uint(t0) * 8388608u);
  r1 = __uint_as_float(__float_as_uint(q1) + __float_as_uint(t1) * 8388608u);
}

}  // namespace ra
