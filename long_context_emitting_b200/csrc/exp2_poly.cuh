// 2^x on the FMA pipe, to share the softmax exponentials with the SFU.
//
// Method: Cody-Waite style range reduction x = n + f with n = round(x),
// obtained by adding and subtracting 1.5 * 2^23 (the sum's low mantissa bits
// hold round(x)), so f lies in [-1/2, 1/2]; 2^f is a degree-5 minimax
// polynomial for RELATIVE error on [-1/2, 1/2], computed for this library with
// the Remez exchange algorithm (gen_exp2_poly.py beside this file prints the
// coefficients) and rounded to float; 2^n is applied by adding n
// to the exponent bits.  Valid for -125 <= x <= 0 after the clamp (smaller x
// returns about 2^-125, which is zero next to a softmax sum >= 1).  Bound
// checked in tests/test_exp2_poly.py (float32 evaluation, Horner with fused
// multiply-add): |relative error| < 3e-7.
#pragma once

#include "f32x2.cuh"

namespace kascade {

// coefficients of 2^f = sum_k c_k f^k, lowest order first
constexpr float kExp2Deg5[6] = {1.0000001192092896f, 0.6931469440460205f, 0.24022120237350464f,
                                0.05550713092088699f, 0.009675540961325169f,
                                0.0013276472454890609f};

// The scalar definition (what the test evaluates).
__device__ __forceinline__ float exp2_poly5(float x) {
  constexpr float c0 = kExp2Deg5[0], c1 = kExp2Deg5[1], c2 = kExp2Deg5[2], c3 = kExp2Deg5[3],
                  c4 = kExp2Deg5[4], c5 = kExp2Deg5[5];
  x = fmaxf(x, -125.f);
  const float t = x + 12582912.f;  // 1.5 * 2^23
  const float n = t - 12582912.f;  // round(x)
  const float f = x - n;
  const float p = fmaf(fmaf(fmaf(fmaf(fmaf(c5, f, c4), f, c3), f, c2), f, c1), f, c0);
  // n sits in the low bits of t (bias 0x4B400000); move it into the exponent
  return __int_as_float(__float_as_int(p) + ((__float_as_int(t) - 0x4B400000) << 23));
}

// exp2_poly5 of two values on packed f32x2 arithmetic: the same operations
// in the same order with the same roundings (t = x + M, n = t - M, f = x - n by
// one fused multiply-add, Horner), so the results are bit-identical to the
// scalar form.  The exponent add uses (t_bits << 23): the bias 0x4B400000
// shifted left by 23 is 0 modulo 2^32.
__device__ __forceinline__ void exp2_poly5_x2(float x0, float x1, float& y0, float& y1) {
  constexpr float c0 = kExp2Deg5[0], c1 = kExp2Deg5[1], c2 = kExp2Deg5[2], c3 = kExp2Deg5[3],
                  c4 = kExp2Deg5[4], c5 = kExp2Deg5[5];
  const uint64_t X = f2_pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t T = f2_add(X, f2_pack(12582912.f, 12582912.f));
  const uint64_t N = f2_add(T, f2_pack(-12582912.f, -12582912.f));
  const uint64_t F = f2_fma(N, f2_pack(-1.f, -1.f), X);
  uint64_t P = f2_fma(f2_pack(c5, c5), F, f2_pack(c4, c4));
  P = f2_fma(P, F, f2_pack(c3, c3));
  P = f2_fma(P, F, f2_pack(c2, c2));
  P = f2_fma(P, F, f2_pack(c1, c1));
  P = f2_fma(P, F, f2_pack(c0, c0));
  float p0, p1, t0, t1;
  f2_unpack(P, p0, p1);
  f2_unpack(T, t0, t1);
  y0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
  y1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
}

}  // namespace kascade
