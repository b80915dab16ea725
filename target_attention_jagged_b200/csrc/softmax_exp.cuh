// 2^x for the attention softmax: on the MUFU (ex2.approx) or, for a share of
// the elements, on the FMA pipe, so that the exponentials of a key tile do not
// all queue on the MUFU (16 results per clock per SM).
//
// The FMA-pipe form, for x <= 8 (a score is at most 8 above the row's running
// maximum, the lazy-rescaling threshold):
//   x = j + f with j = round(x) (by adding and subtracting 1.5 * 2^23) and
//   f in [-1/2, 1/2];
//   2^f by a degree-3 polynomial c0 + c1 f + c2 f^2 + c3 f^3, the minimax
//   approximation for RELATIVE error on [-1/2, 1/2], computed by the Remez
//   exchange algorithm (five alternating extrema of the relative error
//   p(f) / 2^f - 1); its maximum relative error is 7.5e-5, and 7.5e-5 too with
//   the coefficients rounded to fp32 and the polynomial evaluated by fp32 FMAs;
//   2^j is added to the result's exponent bits.
// Below -126 the argument is held at -126: the result is then 2^-126, zero at
// the precision of P (bf16).  Over [-126, 8] the relative error against an
// exact 2^x stays below 1.5e-4 (stca_selftest_ex2 measures it on the device).
#pragma once

#include <stdint.h>

namespace stca {
namespace sx {

constexpr float kMagic = 12582912.0f;          // 1.5 * 2^23
constexpr float kC0 = 0.99992807f, kC1 = 0.69326098f, kC2 = 0.24261112f, kC3 = 0.055171669f;

// MUFU exponential.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA pipe, one element.
__device__ __forceinline__ float ex2_fma(float x) {
  x = fmaxf(x, -126.0f);
  const float t = x + kMagic;                      // round(x) in the low mantissa bits
  const float f = x - (t - kMagic);
  float p = fmaf(f, kC3, kC2);
  p = fmaf(f, p, kC1);
  p = fmaf(f, p, kC0);
  return __uint_as_float(__float_as_uint(p) + (__float_as_uint(t) << 23));
}

// ---- two fp32 lanes per instruction (sm_100 packed f32x2 arithmetic)
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_split(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// 2^x of both lanes on the FMA pipe: the same steps as ex2_fma.
__device__ __forceinline__ void ex2_fma2(float x0, float x1, float& y0, float& y1) {
  const uint64_t magic = f2(kMagic, kMagic);
  const uint64_t x = f2(fmaxf(x0, -126.0f), fmaxf(x1, -126.0f));
  const uint64_t t = f2_add(x, magic);
  const uint64_t f = f2_sub(x, f2_sub(t, magic));
  uint64_t p = f2_fma(f, f2(kC3, kC3), f2(kC2, kC2));
  p = f2_fma(f, p, f2(kC1, kC1));
  p = f2_fma(f, p, f2(kC0, kC0));
  float p0, p1, t0, t1;
  f2_split(p, p0, p1);
  f2_split(t, t0, t1);
  y0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
  y1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
}

// Largest of three (one instruction on sm_100).
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

}  // namespace sx
}  // namespace stca
