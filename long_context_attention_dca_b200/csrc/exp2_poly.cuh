// 2^x on the FMA/ALU pipes, for offloading part of the softmax exponentials
// from the special-function unit (16 results per clock per SM on B200,
// against 128 FMAs per clock).
//
// Method: Cody-Waite style range reduction, x = j + f with j = round(x) and
// f in [-1/2, 1/2], then 2^x = 2^j * p(f) where p is the degree-3 minimax
// (Remez exchange, relative error) polynomial for 2^f on [-1/2, 1/2], fitted
// for this library; max relative error 7.5e-5 evaluated in fp32 (the result
// is rounded to bf16, whose own rounding error is 2^-9 = 2e-3).
//   * round(x) via the 1.5 * 2^23 magic constant: adding it leaves round(x)
//     in the low mantissa bits (valid for |x| < 2^22);
//   * 2^j applied by adding j to the exponent field of p(f).
// Inputs are clamped to >= -125 so the result stays a normal float: it is
// then ~2e-38 instead of exactly 0, which no caller distinguishes.
// Header-only and host-compilable, so its arithmetic can be checked on the
// CPU against std::exp2.
#pragma once

#include <stdint.h>

#include <cmath>
#include <cstring>

#ifdef __CUDACC__
#define DCA_HD __host__ __device__ __forceinline__
#else
#define DCA_HD inline
#endif

namespace dca {

constexpr float kExp2C0 = 0.9999280571937561f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C2 = 0.2426111251115799f;
constexpr float kExp2C3 = 0.0551716685295105f;

DCA_HD int32_t f32_bits(float x) {
#ifdef __CUDA_ARCH__
  return __float_as_int(x);
#else
  int32_t i;
  std::memcpy(&i, &x, 4);
  return i;
#endif
}

DCA_HD float bits_f32(int32_t i) {
#ifdef __CUDA_ARCH__
  return __int_as_float(i);
#else
  float x;
  std::memcpy(&x, &i, 4);
  return x;
#endif
}

DCA_HD float fma32(float a, float b, float c) {
#ifdef __CUDA_ARCH__
  return fmaf(a, b, c);
#else
  return std::fma(a, b, c);
#endif
}

DCA_HD float exp2_poly3(float x) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  x = x > -125.0f ? x : -125.0f;
  const float t = x + kMagic;
  const float r = t - kMagic;            // round(x)
  const float f = x - r;                 // in [-1/2, 1/2]
  float p = fma32(kExp2C3, f, kExp2C2);
  p = fma32(p, f, kExp2C1);
  p = fma32(p, f, kExp2C0);
  const int32_t j = f32_bits(t) - 0x4B400000;  // round(x) as an integer
  return bits_f32(f32_bits(p) + (j << 23));
}

}  // namespace dca
