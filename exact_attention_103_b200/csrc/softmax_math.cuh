// softmax_math.cuh -- the exponential of the forward kernel's softmax on the FMA
// pipe ("FlashAttention V4 deep-dive" (pnsm.cn), section 3.2: part of the
// exponentials computed by a polynomial on the FMA units instead of MUFU ex2),
// in a scalar and a packed two-lane form with identical rounding.
//
// 2^y = 2^j * p(f): j = round(y) by the 1.5*2^23 trick, f = y - j in [-1/2, 1/2],
// p(f) ~ 2^f (our own minimax fit, exp2_poly.h), then 2^j is added to the
// exponent field as an integer (Schraudolph 1999, "A fast, compact approximation
// of the exponential function").  y is clamped below at -125 so the result stays a
// normal float (the exact value there is < 2^-125, far below a bf16 P~).  Valid
// for y <= 64 (the conditional-rescale threshold keeps y <= tau <= 64).
#pragma once
#include <cstdint>

#include "exp2_poly.h"
#include "sm100_ptx.cuh"

namespace attn {

constexpr float kExp2Magic = 12582912.0f;  // 1.5 * 2^23
constexpr float kExp2Clamp = -125.f;

__device__ __forceinline__ float exp2_poly(float y) {
  y = fmaxf(y, kExp2Clamp);
  const float t = y + kExp2Magic;  // rounds y to an integer in t's low bits
  const float f = y - (t - kExp2Magic);
  float p = fmaf(f, ATTN_EXP2_C3, ATTN_EXP2_C2);
  p = fmaf(p, f, ATTN_EXP2_C1);
  p = fmaf(p, f, ATTN_EXP2_C0);
  return __uint_as_float(__float_as_uint(p) + (__float_as_uint(t) << 23));
}

// Two exponentials with f32x2 instructions: the same steps and roundings as
// exp2_poly, lane by lane, in about half the issue slots.
__device__ __forceinline__ void exp2_poly_x2(float& y0, float& y1) {
  y0 = fmaxf(y0, kExp2Clamp);
  y1 = fmaxf(y1, kExp2Clamp);
  float t0, t1, j0, j1, f0, f1, p0, p1;
  fadd2_bc(t0, t1, y0, y1, kExp2Magic);
  fsub2_bc(j0, j1, t0, t1, kExp2Magic);
  fsub2(f0, f1, y0, y1, j0, j1);
  ffma2_bc(p0, p1, f0, f1, ATTN_EXP2_C3, ATTN_EXP2_C2);
  ffma2_vb(p0, p1, p0, p1, f0, f1, ATTN_EXP2_C1);
  ffma2_vb(p0, p1, p0, p1, f0, f1, ATTN_EXP2_C0);
  y0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
  y1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
}

}  // namespace attn
