// 2^x on the FMA pipes, for a share of the softmax exponentials (the MUFU unit
// retires 16 exponentials per clock per SM, which alone would cap the tensor
// cores near their speed).
//
// Method: round-to-nearest range reduction, x = i + f with i = rint(x) and
// f in [-1/2, 1/2] (the integer comes out of adding 1.5 * 2^23, which leaves
// rint(x) in the low mantissa bits), a degree-3 polynomial for 2^f, and the
// exponent i added straight into the result's exponent field.  The
// coefficients are a relative-error minimax fit of 2^f on [-1/2, 1/2]
// (Lawson-reweighted least squares on Chebyshev nodes), derived by
// paged_kv_cache_exact_b200/exp2_fit.py; max relative error 7.5e-5, far
// below half an ulp of the bf16 P it feeds (2^-9).  x is clamped below at
// -125 so the exponent never wraps; 2^-125 stands in for smaller results.
#pragma once

#include "sm100_ptx.cuh"

namespace pkv {
namespace sm100 {

constexpr float kExp2C0 = 0.9999280571937561f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C2 = 0.2426111251115799f;
constexpr float kExp2C3 = 0.0551716648042202f;
constexpr float kRoundMagic = 12582912.0f;   // 1.5 * 2^23

// 2^x for a pair (x0, x1) packed in f32x2.
PKV_DEVINLINE void exp2_poly_pair(uint64_t x, float& y0, float& y1) {
  float a, b;
  unf2(x, a, b);
  a = fmaxf(a, -125.f);
  b = fmaxf(b, -125.f);
  const uint64_t xc = f2(a, b);
  const uint64_t magic = f2(kRoundMagic, kRoundMagic);
  const uint64_t t = add2(xc, magic);            // low mantissa bits hold rint(x)
  const uint64_t r = sub2(t, magic);             // rint(x) as a float
  const uint64_t fr = sub2(xc, r);               // f in [-1/2, 1/2]
  uint64_t p = fma2(f2(kExp2C3, kExp2C3), fr, f2(kExp2C2, kExp2C2));
  p = fma2(p, fr, f2(kExp2C1, kExp2C1));
  p = fma2(p, fr, f2(kExp2C0, kExp2C0));
  float p0, p1, t0, t1;
  unf2(p, p0, p1);
  unf2(t, t0, t1);
  y0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
  y1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}

}  // namespace sm100
}  // namespace pkv
