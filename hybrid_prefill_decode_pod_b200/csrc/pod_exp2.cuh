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

}  // namespace pod
