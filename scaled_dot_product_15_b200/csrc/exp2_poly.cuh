// 2^x on the FMA pipe, for the share of the softmax exponentials that the
// multi-function unit (16 results per clock per SM) cannot absorb.
//
// Method: Cody-Waite style range reduction x = j + f with j = floor(x) and
// f in [0, 1), then 2^f from a degree-3 minimax polynomial (minimised
// relative error on [0, 1], found by a Remez exchange; fit_exp2_poly.py
// reproduces the coefficients), and 2^j applied by adding j to the float's
// exponent field.  floor(x) comes from one add rounded toward -inf to
// 1.5 * 2^23, whose last mantissa bits then hold the integer.
// Maximum relative error 7.5e-5 (float32 evaluation), well under half an ulp
// of the fp16 / bf16 weights it feeds.  x is clamped below at -126 so the
// exponent field never underflows; NaN propagates.
#pragma once

#include <stdint.h>

namespace sdpa15 {
namespace exp2poly {

constexpr float kC0 = 0.9999251961708069f;
constexpr float kC1 = 0.6958335638046265f;
constexpr float kC2 = 0.22606715559959412f;
constexpr float kC3 = 0.07802452147006989f;
constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
constexpr float kMinX = -126.0f;

__device__ __forceinline__ uint64_t pk(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void upk(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fadd2_rm(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rm.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float max_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

// 2^x0, 2^x1 for a pair held as two floats.
__device__ __forceinline__ void exp2_pair(float x0, float x1, float& y0, float& y1) {
  const uint64_t x = pk(max_nan(x0, kMinX), max_nan(x1, kMinX));
  const uint64_t t = fadd2_rm(x, pk(kMagic, kMagic));          // 1.5*2^23 + floor(x)
  const uint64_t j = fadd2(t, pk(-kMagic, -kMagic));          // floor(x), exact
  const uint64_t f = ffma2(j, pk(-1.f, -1.f), x);              // x - floor(x) in [0, 1)
  uint64_t p = ffma2(pk(kC3, kC3), f, pk(kC2, kC2));
  p = ffma2(p, f, pk(kC1, kC1));
  p = ffma2(p, f, pk(kC0, kC0));
  float p0, p1, t0, t1;
  upk(p, p0, p1);
  upk(t, t0, t1);
  // The low bits of t hold floor(x) in two's complement; shifted into the
  // exponent field they scale p by 2^floor(x) (1.5*2^23's own bits shift out).
  y0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
  y1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
}

}  // namespace exp2poly
}  // namespace sdpa15
