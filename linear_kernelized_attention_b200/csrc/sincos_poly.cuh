// sincos_poly.cuh - sine and cosine on the FMA pipe, for the trig feature map.
//
// The trig feature map of the explainer page "用随机特征“骗”过 softmax，Transformer 注意力也能跑成线性？"
// (section 核心机制：FAVOR+, cos/sin pairs) needs cos(u) and sin(u) of every projected angle. The
// SFU (MUFU) evaluates them at 16 results per SM per clock, which would bound the trig kernels;
// the FMA pipe runs 128 lanes per SM per clock. The kernels therefore evaluate a fixed share of
// the angles with the polynomials below and the rest with the SFU's approximate sin/cos.
//
// Reduction: n = round(u / pi), r = u - n pi in [-pi/2, pi/2] with pi = kPiHi + kPiLo (Cody and
// Waite); sin u = (-1)^n sin r, cos u = (-1)^n cos r. The rounding to an integer adds 1.5 * 2^23,
// whose unit in the last place is 1, so n's parity is the low bit of the sum's bit pattern.
// n * kPiHi is exact for |n| < 256 (|u| < 800).
// Approximation: minimax (Remez exchange) polynomials on [-pi/2, pi/2],
//   sin r = r + r^3 (kS1 + kS2 r^2 + kS3 r^4),  cos r = 1 + r^2 (kC1 + kC2 r^2 + kC3 r^4 + kC4 r^6).
// The coefficients are derived by sincos_coeffs.py beside this file; their float32 evaluation
// errs by at most 1e-6 (sin) and 2e-7 (cos) in absolute value for |u| <= 400, below the 16-bit
// rounding (>= 2^-12 relative) the features then take. 16 FMA-pipe instructions give both values.
#pragma once
#include <cstdint>

namespace favor {

constexpr float kPiHi = 3.141601562e+00f, kPiLo = -8.908909876e-06f;
constexpr float kInvPi = 0.318309886183790671538f;
constexpr float kS1 = -1.666568071e-01f, kS2 = 8.312365972e-03f, kS3 = -1.849218097e-04f;
constexpr float kC1 = -4.999993145e-01f, kC2 = 4.166398942e-02f, kC3 = -1.385592739e-03f, kC4 = 2.319438681e-05f;

__device__ __forceinline__ void sincos_fma(float u, float& s, float& c) {
  const float t = __fmaf_rn(u, kInvPi, 12582912.0f);
  const float n = __fsub_rn(t, 12582912.0f);
  float r = __fmaf_rn(n, -kPiHi, u);
  r = __fmaf_rn(n, -kPiLo, r);
  const float r2 = __fmul_rn(r, r);
  float ps = __fmaf_rn(r2, kS3, kS2);
  ps = __fmaf_rn(r2, ps, kS1);
  const float r3 = __fmul_rn(r2, r);
  const float sr = __fmaf_rn(r3, ps, r);
  float pc = __fmaf_rn(r2, kC4, kC3);
  pc = __fmaf_rn(r2, pc, kC2);
  pc = __fmaf_rn(r2, pc, kC1);
  const float cr = __fmaf_rn(r2, pc, 1.0f);
  const uint32_t sgn = __float_as_uint(t) << 31;
  s = __uint_as_float(__float_as_uint(sr) ^ sgn);
  c = __uint_as_float(__float_as_uint(cr) ^ sgn);
}

// SFU path: the hardware's approximate sine and cosine (sin.approx / cos.approx).
__device__ __forceinline__ void sincos_sfu(float u, float& s, float& c) { __sincosf(u, &s, &c); }

// Angle j of a group of 8 takes the FMA path when bit j of kPolyMask is set. The mask sets the
// share of angles moved off the SFU; it is a compile-time constant so the unrolled loops carry
// no branch.
template <uint32_t kPolyMask>
__device__ __forceinline__ void sincos_mixed(int j, float u, float& s, float& c) {
  if ((kPolyMask >> (j & 7)) & 1u)
    sincos_fma(u, s, c);
  else
    sincos_sfu(u, s, c);
}

}  // namespace favor
