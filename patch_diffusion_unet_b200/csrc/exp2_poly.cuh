// 2^x on the FMA pipe for pairs of fp32 values (packed f32x2 arithmetic), used by the
// attention softmax to take part of its exponentials off the MUFU unit.
//
// Range reduction x = j + f with j = rint(x) (magic-constant rounding: adding 1.5 * 2^23
// leaves j in the low mantissa bits), |f| <= 1/2; 2^f by a degree-3 polynomial; 2^j added
// into the exponent field of the result.  The coefficients are the minimax fit in relative
// error on [-1/2, 1/2] by Lawson's algorithm (iteratively reweighted least squares on 256
// Chebyshev nodes), max relative error 7.48e-5; exp2_poly_fit.py next to this file derives
// them.  x is clamped to >= -125 so the exponent cannot wrap (2^-125 stands for anything
// smaller, which is negligible next to a softmax row's maximum term of 1).
#pragma once
#include <stdint.h>

namespace dfp {

__device__ __forceinline__ uint64_t f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_split(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// 2^x for both lanes of x2, as fp32 bit patterns (r0: first lane).
__device__ __forceinline__ void ex2_poly_pair_f32(uint64_t x2, uint32_t& r0, uint32_t& r1) {
  float x0, x1;
  f2_split(x2, x0, x1);
  const uint64_t x = f2(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t t = add2(x, f2(12582912.f, 12582912.f));
  const uint64_t j = add2(t, f2(-12582912.f, -12582912.f));
  const uint64_t f = fma2(j, f2(-1.f, -1.f), x);
  uint64_t p = fma2(f2(0.0551716648f, 0.0551716648f), f, f2(0.242611125f, 0.242611125f));
  p = fma2(p, f, f2(0.693260968f, 0.693260968f));
  p = fma2(p, f, f2(0.999928057f, 0.999928057f));
  float p0, p1, t0, t1;
  f2_split(p, p0, p1);
  f2_split(t, t0, t1);
  r0 = __float_as_uint(p0) + (__float_as_uint(t0) << 23);
  r1 = __float_as_uint(p1) + (__float_as_uint(t1) << 23);
}

// The same pair truncated to bf16 (upper halves; lo = first lane).
__device__ __forceinline__ uint32_t ex2_poly_pair_bf16(uint64_t x2) {
  uint32_t r0, r1, r;
  ex2_poly_pair_f32(x2, r0, r1);
  asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(r) : "r"(r0), "r"(r1));
  return r;
}

}  // namespace dfp
