// 2^x on the FMA pipe, for exponents of softmax terms (x <= 0), two lanes per instruction.
//
// The tensor-core attention needs two exponentials per score (row statistics, then probabilities),
// more than the 16-per-clock multi-function unit of an SM delivers next to the tensor cores, so a
// fixed share of them is computed here instead, on the paired float32 FMA units.
//
// Method: Cody-Waite range reduction x = j + f with j = rint(x) and f in [-1/2, 1/2] (the add of
// 1.5 * 2^23 rounds x to an integer held in the low mantissa bits of the sum), then 2^f by a
// degree-5 minimax polynomial of 2^f on [-1/2, 1/2] in relative error (Remez exchange algorithm),
// its constant term then set to exactly 1 (so 2^j is exact at integers) and the other coefficients,
// rounded to float32, adjusted ulp by ulp to the smallest maximum relative error (1.14e-7 in exact
// arithmetic; 1.8e-7 with the float32 roundings of the Horner steps).
// The factor 2^j enters as an integer add of j << 23 to the result's exponent field.
// x is clamped to [-126, +inf): the result is then at least 2^-126 (the smallest normal float)
// where the flush-to-zero ex2 instruction would return 0; every exponent used here is <= 0 up to
// rounding, so j <= 0 and the exponent field stays in range.
#pragma once

#include <stdint.h>

namespace spt {

__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  constexpr float kRound = 12582912.0f;   // 1.5 * 2^23
  x.x = fmaxf(x.x, -126.0f);
  x.y = fmaxf(x.y, -126.0f);
  const float2 t = __fadd2_rn(x, make_float2(kRound, kRound));            // rint(x) + 1.5 * 2^23
  const float2 j = __fadd2_rn(t, make_float2(-kRound, -kRound));          // rint(x), exact
  const float2 f = __ffma2_rn(j, make_float2(-1.0f, -1.0f), x);          // x - j in [-1/2, 1/2], exact
  float2 p = __ffma2_rn(make_float2(1.32765993476e-03f, 1.32765993476e-03f), f,
                        make_float2(9.67559963465e-03f, 9.67559963465e-03f));
  p = __ffma2_rn(p, f, make_float2(5.55074438453e-02f, 5.55074438453e-02f));
  p = __ffma2_rn(p, f, make_float2(2.40221768618e-01f, 2.40221768618e-01f));
  p = __ffma2_rn(p, f, make_float2(6.93146944046e-01f, 6.93146944046e-01f));
  p = __ffma2_rn(p, f, make_float2(1.0f, 1.0f));
  // the low bits of t's pattern hold j (two's complement); shifted to the exponent field the
  // offset of the rounding constant drops out
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

}  // namespace spt
