// softmax.cuh -- pieces of the attention softmax shared by the FP8 and fp16
// kernels: key masking of a ragged tile, and 2^x split between the MUFU
// (ex2.approx) and the FMA pipe (range reduction + Remez polynomial).
#pragma once
#include <math.h>
#include <stdint.h>

#include "exp2_poly.cuh"
#include "ptx.cuh"

namespace sdm {

// Keys at or past `nvalid` (counted from the tile start) get logit -inf, so
// they neither raise the max nor receive probability.
__device__ __forceinline__ void mask_keys(uint32_t (&ra)[32], uint32_t (&rb)[32], int col0, int64_t nvalid) {
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    if (col0 + i >= nvalid) ra[i] = __float_as_uint(-INFINITY);
    if (col0 + 32 + i >= nvalid) rb[i] = __float_as_uint(-INFINITY);
  }
}

// 2^t on the FMA pipe for a pair of lanes: t = j + f with j = round(t) (the
// 1.5*2^23 rounding trick), f in [-1/2, 1/2], 2^f from the degree-4 Remez
// polynomial of exp2_poly.cuh (relative error < 3e-6), and 2^j added to the
// exponent field.  t is clamped at kClamp first, which keeps the exponent
// arithmetic in range (kClamp >= -125 gives a normal fp32 result).  The FP8
// kernel clamps at -30: every result below 2^-10 is an e4m3 zero anyway.
template <int kClamp = -30>
__device__ __forceinline__ void exp2_fma2(float t0, float t1, float& p0, float& p1) {
  static_assert(kClamp >= -125 && kClamp <= 0, "clamp keeps 2^j a normal float");
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  t0 = fmaxf(t0, static_cast<float>(kClamp));
  t1 = fmaxf(t1, static_cast<float>(kClamp));
  float r0, r1, j0, j1, f0, f1;
  add2(r0, r1, t0, t1, kRound, kRound);
  sub2(j0, j1, r0, r1, kRound, kRound);
  sub2(f0, f1, t0, t1, j0, j1);
  float q0 = kExp2C4, q1 = kExp2C4;
  fma2(q0, q1, q0, q1, f0, f1, kExp2C3, kExp2C3);
  fma2(q0, q1, q0, q1, f0, f1, kExp2C2, kExp2C2);
  fma2(q0, q1, q0, q1, f0, f1, kExp2C1, kExp2C1);
  fma2(q0, q1, q0, q1, f0, f1, kExp2C0, kExp2C0);
  // the bit pattern of r holds j + 1.5*2^23; shifted by 23 the constant part
  // vanishes modulo 2^32, leaving j in the exponent field
  p0 = __uint_as_float(__float_as_uint(q0) + (__float_as_uint(r0) << 23));
  p1 = __uint_as_float(__float_as_uint(q1) + (__float_as_uint(r1) << 23));
}

// Which of the 8 four-key words of a 32-key chunk take the FMA-pipe 2^x:
// kPolyEighths of them, spread evenly; the others use the MUFU ex2.
#ifndef SDM_POLY_EIGHTHS
#define SDM_POLY_EIGHTHS 2
#endif
constexpr int kPolyEighths = SDM_POLY_EIGHTHS;
__host__ __device__ constexpr bool poly_word(int w) {
  return (w * kPolyEighths) / 8 != ((w + 1) * kPolyEighths) / 8;
}

}  // namespace sdm
