// exp2_poly.cuh -- 2^t on the FMA pipe, for the share of the softmax
// exponentials that the attention kernels take off the SFU.
//
// The exp pass of the attention kernels issues one SFU ex2 per score, and
// the SFU retires 16 of them per clock per SM (the kernels' throughput
// floor); the FP32 pipes sit partly idle meanwhile.  A fixed share of the
// scores is therefore evaluated here instead, two at a time with the packed
// FP32x2 instructions:
//   t = j + f, j = rint(t) (the 1.5 * 2^23 add leaves j in the low mantissa
//   bits), f = t - j in [-1/2, 1/2] (exact);
//   2^f by a degree-4 polynomial in Horner form (coefficients from a Remez
//   exchange on the relative error over [-1/2, 1/2]: fit_exp2_poly.py);
//   2^t = 2^f with j added to its exponent field (an integer add of j << 23).
// Maximum relative error 2.7e-6 (2^-18.5) over the reduced range, FP32
// Horner rounding included; ex2.approx.f32 is of the same order (2^-22).
// t is clamped at -125 so that 2^j stays a normal number (2^-125 is far
// below the smallest P~ code and changes no row sum measurably).
#pragma once

namespace sage {

// Coefficients c0..c4 of 2^f ~ c0 + c1 f + c2 f^2 + c3 f^3 + c4 f^4 on
// [-1/2, 1/2] (FP32 bit patterns written by fit_exp2_poly.py).
constexpr unsigned kExp2C0 = 0x3f7ffff4u;
constexpr unsigned kExp2C1 = 0x3f31706eu;
constexpr unsigned kExp2C2 = 0x3e76036du;
constexpr unsigned kExp2C3 = 0x3d650a20u;
constexpr unsigned kExp2C4 = 0x3c1ccbebu;

// 2^t for both lanes of t (t <= 128).
__device__ __forceinline__ float2 exp2_poly2(float2 t) {
  const float2 kM = make_float2(12582912.f, 12582912.f);    // 1.5 * 2^23
  const float2 kMn = make_float2(-12582912.f, -12582912.f);
  t.x = fmaxf(t.x, -125.f);
  t.y = fmaxf(t.y, -125.f);
  const float2 y = __fadd2_rn(t, kM);    // 1.5 * 2^23 + rint(t), exactly
  const float2 j = __fadd2_rn(y, kMn);   // rint(t)
  const float2 f = __fadd2_rn(t, make_float2(-j.x, -j.y));  // t - rint(t), exact
  const float2 c4 = make_float2(__uint_as_float(kExp2C4), __uint_as_float(kExp2C4));
  const float2 c3 = make_float2(__uint_as_float(kExp2C3), __uint_as_float(kExp2C3));
  const float2 c2 = make_float2(__uint_as_float(kExp2C2), __uint_as_float(kExp2C2));
  const float2 c1 = make_float2(__uint_as_float(kExp2C1), __uint_as_float(kExp2C1));
  const float2 c0 = make_float2(__uint_as_float(kExp2C0), __uint_as_float(kExp2C0));
  float2 p = __ffma2_rn(c4, f, c3);
  p = __ffma2_rn(p, f, c2);
  p = __ffma2_rn(p, f, c1);
  p = __ffma2_rn(p, f, c0);
  // the low 9 bits of y's pattern hold j (two's complement): j << 23 mod 2^32
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(y.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(y.y) << 23)));
}

}  // namespace sage
