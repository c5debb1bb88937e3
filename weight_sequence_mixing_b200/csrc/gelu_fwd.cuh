// GELU(x) = x Phi(x) alone, without its derivative (the apply's hidden layer), with erf from
// Abramowitz & Stegun, Handbook of Mathematical Functions, formula 7.1.28:
//   erf(u) = 1 - (1 + a1 u + a2 u^2 + a3 u^3 + a4 u^4 + a5 u^5 + a6 u^6)^-16,  u >= 0,
// absolute error <= 3e-7.  It takes one reciprocal and no exponential per value; 7.1.26
// (epilogues.cuh), used where the density is needed too, takes a reciprocal and an
// exponential.  The coefficients are the published ones, with u = |x| / sqrt 2 folded in
// (b_k = a_k 2^(-k/2)); Phi(-|x|) = (1 - erf(u)) / 2.  The reciprocal's relative error
// (about 2^-23) grows sixteenfold in the power: still far below the bf16 rounding of H.
#pragma once
#include "epilogues.cuh"

namespace ttt {

namespace normal_as28 {
constexpr double kS = 0.70710678118654752;  // 1 / sqrt 2
constexpr float kB1 = float(0.0705230784 * kS), kB2 = float(0.0422820123 * kS * kS),
                kB3 = float(0.0092705272 * kS * kS * kS), kB4 = float(0.0001520143 * kS * kS * kS * kS),
                kB5 = float(0.0002765672 * kS * kS * kS * kS * kS),
                kB6 = float(0.0000430638 * kS * kS * kS * kS * kS * kS);
}  // namespace normal_as28

// two GELUs at once, multiplies and adds as paired fp32 instructions
__device__ __forceinline__ float2 gelu_fwd2(float2 x) {
  using namespace normal_as28;
  const float2 u = make_float2(fabsf(x.x), fabsf(x.y));
  float2 p = fma2(make_float2(kB6, kB6), u, make_float2(kB5, kB5));
  p = fma2(p, u, make_float2(kB4, kB4));
  p = fma2(p, u, make_float2(kB3, kB3));
  p = fma2(p, u, make_float2(kB2, kB2));
  p = fma2(p, u, make_float2(kB1, kB1));
  p = fma2(p, u, make_float2(1.0f, 1.0f));
  const float2 r = make_float2(rcp_approx(p.x), rcp_approx(p.y));
  const float2 r2 = mul2(r, r), r4 = mul2(r2, r2), r8 = mul2(r4, r4);
  const float2 q = mul2(mul2(r8, r8), make_float2(0.5f, 0.5f));  // Phi(-|x|)
  const float2 cdf = make_float2(x.x >= 0.0f ? 1.0f - q.x : q.x, x.y >= 0.0f ? 1.0f - q.y : q.y);
  return mul2(x, cdf);
}

}  // namespace ttt
