// Packed fp32 pairs (sm_100 f32x2 arithmetic) and the FMA-pipe exponential
// used by the attention softmax. Device-only helpers, header so that a test
// kernel can check the exponential against the hardware's on the GPU.
#pragma once

#include <stdint.h>

namespace sda {

__device__ __forceinline__ uint64_t f2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_split(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x for a pair, on the FMA pipe (Cody-Waite style split x = j + f with
// j = floor(x), f in [0, 1), then 2^f from a cubic with p(0) = 1 whose other
// coefficients minimise the maximum relative error on [0, 1) (Lawson-weighted
// least squares; max relative error 8.6e-5, below the bf16 rounding of P).
// j is read out of the float t = 1.5 * 2^23 + j (round-down add) and added
// to the exponent field. Inputs are clamped to [-127, ...): callers use it on
// finite arguments only (full blocks carry no -inf mask).
constexpr float kPoly1 = 0.69511634f, kPoly2 = 0.227647f, kPoly3 = 0.0770652f;
__device__ __forceinline__ void ex2_fma2(float x0, float x1, float& p0, float& p1) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  x0 = fmaxf(x0, -127.f);
  x1 = fmaxf(x1, -127.f);
  const float t0 = __fadd_rd(x0, kMagic), t1 = __fadd_rd(x1, kMagic);
  const uint64_t j2 = add2(f2(t0, t1), f2(-kMagic, -kMagic));       // floor(x), exact
  const uint64_t fr = fma2(j2, f2(-1.f, -1.f), f2(x0, x1));          // x - floor(x)
  uint64_t p = fma2(f2(kPoly3, kPoly3), fr, f2(kPoly2, kPoly2));
  p = fma2(p, fr, f2(kPoly1, kPoly1));
  p = fma2(p, fr, f2(1.f, 1.f));
  float q0, q1;
  f2_split(p, q0, q1);
  p0 = __uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23));
  p1 = __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23));
}

}  // namespace sda
