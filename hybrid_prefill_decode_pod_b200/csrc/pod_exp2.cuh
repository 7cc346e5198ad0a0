// pod_exp2.cuh -- 2^x on the FMA/integer pipes, for part of the softmax.
//
// On B200 one MUFU.EX2 per score element costs as much SM time as both MMAs
// of that element, so the prefill softmax evaluates a share of its
// exponentials here instead and leaves the rest to ex2.approx.
//
// Method (Cody & Waite, "Software Manual for the Elementary Functions", 1980:
// reduce the argument by an integer, approximate the remainder, rescale):
//   n = round(x) via the 1.5 * 2^23 shifter (float add rounds to an integer),
//   f = x - n in [-0.5, 0.5] (exact),
//   2^f ~ c0 + c1 f + c2 f^2 + c3 f^3, coefficients fitted for relative error
//   by fit_exp2_poly.py next to this file (worst relative error 7.5e-5),
//   2^x = 2^f * 2^n by adding n to the exponent field.
// Valid for finite x <= 126; x is clamped below at -125 so the result stays a
// normal float (2^-125 instead of smaller values, which are far below the
// rounding of the row's largest weight). Callers never pass -inf here.
#pragma once
#include <stdint.h>
#include <string.h>

#ifndef __CUDACC__
#define POD_HD inline
#else
#define POD_HD __host__ __device__ __forceinline__
#endif

namespace pod {

constexpr float kExp2C0 = 9.999280572e-01f;
constexpr float kExp2C1 = 6.932609677e-01f;
constexpr float kExp2C2 = 2.426111400e-01f;
constexpr float kExp2C3 = 5.517165735e-02f;

POD_HD int32_t f2i_bits(float x) {
#ifdef __CUDA_ARCH__
  return __float_as_int(x);
#else
  int32_t i;
  memcpy(&i, &x, 4);
  return i;
#endif
}
POD_HD float i2f_bits(int32_t i) {
#ifdef __CUDA_ARCH__
  return __int_as_float(i);
#else
  float x;
  memcpy(&x, &i, 4);
  return x;
#endif
}

POD_HD float exp2_poly(float x) {
  x = x < -125.0f ? -125.0f : x;
  const float shifter = 12582912.0f;  // 1.5 * 2^23
  const float t = x + shifter;         // round(x) sits in the low mantissa bits of t
  const float f = x - (t - shifter);   // exact, in [-0.5, 0.5]
#ifdef __CUDA_ARCH__
  float p = fmaf(kExp2C3, f, kExp2C2);
  p = fmaf(p, f, kExp2C1);
  p = fmaf(p, f, kExp2C0);
#else
  float p = __builtin_fmaf(kExp2C3, f, kExp2C2);
  p = __builtin_fmaf(p, f, kExp2C1);
  p = __builtin_fmaf(p, f, kExp2C0);
#endif
  // bits(t) = bits(shifter) + round(x), and bits(shifter) * 2^23 vanishes
  // modulo 2^32, so bits(t) * 2^23 adds round(x) to p's exponent field.
  return i2f_bits((int32_t)((uint32_t)f2i_bits(p) + (uint32_t)f2i_bits(t) * 8388608u));
}

#ifdef __CUDACC__
// exp2_poly on both halves of a packed pair with f32x2 instructions. Every
// step is the scalar version's operation, rounded the same way, so each half
// equals exp2_poly of that half (f = x - n by one fused multiply-add, exact
// like the scalar subtraction since |f| <= 0.5).
__device__ __forceinline__ uint64_t exp2_poly2(float x0, float x1) {
  x0 = fmaxf(x0, -125.0f);
  x1 = fmaxf(x1, -125.0f);
  const float shifter = 12582912.0f;  // 1.5 * 2^23
  uint64_t x, t, n, f, p, c;
  asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(x0), "f"(x1));
  asm("mov.b64 %0, {%1, %1};" : "=l"(c) : "f"(shifter));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(t) : "l"(x), "l"(c));  // t = x + shifter
  asm("mov.b64 %0, {%1, %1};" : "=l"(c) : "f"(-shifter));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(n) : "l"(t), "l"(c));  // n = round(x)
  asm("mov.b64 %0, {%1, %1};" : "=l"(c) : "f"(-1.0f));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(f) : "l"(n), "l"(c), "l"(x));  // f = x - n
  uint64_t c3, c2;
  asm("mov.b64 %0, {%1, %1};" : "=l"(c3) : "f"(kExp2C3));
  asm("mov.b64 %0, {%1, %1};" : "=l"(c2) : "f"(kExp2C2));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(p) : "l"(c3), "l"(f), "l"(c2));
  asm("mov.b64 %0, {%1, %1};" : "=l"(c) : "f"(kExp2C1));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(p) : "l"(p), "l"(f), "l"(c));
  asm("mov.b64 %0, {%1, %1};" : "=l"(c) : "f"(kExp2C0));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(p) : "l"(p), "l"(f), "l"(c));
  uint32_t p0, p1, t0, t1;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(p0), "=r"(p1) : "l"(p));
  asm("mov.b64 {%0, %1}, %2;" : "=r"(t0), "=r"(t1) : "l"(t));
  const uint32_t r0 = p0 + t0 * 8388608u, r1 = p1 + t1 * 8388608u;
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(r0), "r"(r1));
  return r;
}
#endif

}  // namespace pod
