// HoPE rotation shared by the pre-pass (hope.cu) and the kernels that rotate
// their query tiles on the fly (select_sm100.cu, attn_sm100.cu), so that both
// routes give the same bits (molayo1419.me, "Engineering details", HoPE:
// rotary embedding on the dimensions inside the pre-training window, none on
// the others).  Dimensions pair up as (i, i + d/2); pair i < npairs turns by
// (pos0 + t) * theta_i, theta_i = base^(-2i/d) (formed once on the host in
// double precision).  The angle a = pos * theta_i is reduced by pi/2 in
// double precision (Cody-Waite, pi/2 split into two doubles: a reaches ~4e6
// rad at 4M tokens, where an fp32 angle would be off by tenths of a radian)
// to x in [-pi/4, pi/4] and a quadrant; sin x and cos x are the Taylor
// series through x^9 and x^10 (remainders below 2e-9 and 2e-10 on that
// interval) evaluated by Horner's rule in fp32 with fused multiply-adds, and
// the quadrant maps them to sin a, cos a.  Branch-free, so the 8 pairs a
// thread handles per step overlap.  The rotation itself is fp32 with every
// product and sum rounded separately.
#pragma once

#include <cuda_runtime.h>

namespace hils {

constexpr int kHopeMaxPairs = 64;

struct HopeParams {
  int npairs;  // rotated pairs (0: no rotation)
  int pos0;    // position of row 0
  double theta[kHopeMaxPairs];
};

// theta_i for pairs 0 .. npairs-1 (host)
inline HopeParams hope_params(int d, int npairs, int pos0, double base);

#ifdef __CUDACC__
// pi/2 as a sum of two doubles (Cody-Waite reduction)
constexpr double kHopeHalfPiHi = 1.5707963267948966;
constexpr double kHopeHalfPiLo = 6.123233995736766e-17;
constexpr double kHopeTwoOverPi = 0.6366197723675814;
// 1.5 * 2^52: adding it rounds a double in [0, 2^51) to an integer held in
// the low mantissa bits
constexpr double kHopeRoundMagic = 6755399441055744.0;

__device__ __forceinline__ void hope_sincos(double theta, long long pos, float &sn, float &cs) {
  const double a = (double)pos * theta;  // >= 0, below 2^31
  const double kd = fma(a, kHopeTwoOverPi, kHopeRoundMagic);  // nearest integer k to 2a/pi
  const double k = kd - kHopeRoundMagic;
  const float x = (float)fma(-k, kHopeHalfPiLo, fma(-k, kHopeHalfPiHi, a));
  const float x2 = __fmul_rn(x, x);
  // sin x = x (1 - x^2/3! + x^4/5! - x^6/7! + x^8/9!)
  float s = __fmaf_rn(x2, 1.0f / 362880.0f, -1.0f / 5040.0f);
  s = __fmaf_rn(x2, s, 1.0f / 120.0f);
  s = __fmaf_rn(x2, s, -1.0f / 6.0f);
  s = __fmaf_rn(__fmul_rn(x2, x), s, x);
  // cos x = 1 - x^2/2! + x^4/4! - x^6/6! + x^8/8! - x^10/10!
  float c = __fmaf_rn(x2, -1.0f / 3628800.0f, 1.0f / 40320.0f);
  c = __fmaf_rn(x2, c, -1.0f / 720.0f);
  c = __fmaf_rn(x2, c, 1.0f / 24.0f);
  c = __fmaf_rn(x2, c, -0.5f);
  c = __fmaf_rn(x2, c, 1.0f);
  // a = x + q pi/2: (sin, cos) = (s, c), (c, -s), (-s, -c), (-c, s) for q = 0..3
  const int q = __double2loint(kd) & 3;  // k mod 4
  const float s1 = (q & 1) ? c : s, c1 = (q & 1) ? s : c;
  sn = (q & 2) ? -s1 : s1;
  cs = ((q + 1) & 2) ? -c1 : c1;
}

// (x_i, x_{i+d/2}) turned by the angle whose sine and cosine are sn, cs
__device__ __forceinline__ void hope_rotate(float xi, float xj, float sn, float cs, float &yi,
                                            float &yj) {
  yi = __fsub_rn(__fmul_rn(xi, cs), __fmul_rn(xj, sn));
  yj = __fadd_rn(__fmul_rn(xi, sn), __fmul_rn(xj, cs));
}
#endif

}  // namespace hils

#include <cmath>

inline hils::HopeParams hils::hope_params(int d, int npairs, int pos0, double base) {
  HopeParams hp{};
  hp.npairs = npairs;
  hp.pos0 = pos0;
  const double lb = std::log2(base);
  for (int i = 0; i < npairs && i < kHopeMaxPairs; ++i) hp.theta[i] = std::exp2(-(2.0 * i / d) * lb);
  return hp;
}
