// Packed fp32 pair arithmetic and a polynomial 2^x on the FMA pipe, shared by
// the attention kernel and its diagnostic entry point.
#pragma once

#include <cstdint>

namespace wf {

// Packed pairs of fp32 in one 64-bit register (sm_100 f32x2 arithmetic).
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unf2(uint64_t v, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// 2^x for a pair, on the FMA pipe instead of the MUFU unit, by Cody-Waite
// style range reduction: x = n + f with n = round(x) (taken from the low
// mantissa bits of x + 1.5 * 2^23) and f in [-1/2, 1/2]; 2^f from a degree-3
// polynomial fitted (Remez exchange on the relative error) to 2^f on
// [-1/2, 1/2], max relative error 7.5e-5, far below the 2^-9 half-ulp of the
// bf16 P it feeds; 2^n is added to the exponent field. x < -126 (including
// the -inf of masked keys) gives 0.
__device__ __forceinline__ uint64_t ex2_poly2(uint64_t x2) {
  constexpr float kShift = 12582912.0f;              // 1.5 * 2^23
  constexpr float c0 = 0.9999280571937561f, c1 = 0.6932609677314758f;
  constexpr float c2 = 0.2426111251115799f, c3 = 0.0551716685295105f;
  float x0, x1;
  unf2(x2, x0, x1);
  const bool z0 = x0 < -126.0f, z1 = x1 < -126.0f;
  const uint64_t xc = f2(fmaxf(x0, -126.0f), fmaxf(x1, -126.0f));
  const uint64_t t = fadd2(xc, f2(kShift, kShift));
  const uint64_t f = ffma2(fadd2(t, f2(-kShift, -kShift)), f2(-1.0f, -1.0f), xc);
  uint64_t q = ffma2(f2(c3, c3), f, f2(c2, c2));
  q = ffma2(q, f, f2(c1, c1));
  q = ffma2(q, f, f2(c0, c0));
  float t0, t1, q0, q1;
  unf2(t, t0, t1);
  unf2(q, q0, q1);
  q0 = z0 ? 0.0f : __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
  q1 = z1 ? 0.0f : __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
  return f2(q0, q1);
}

}  // namespace wf
