// HoPE rotation shared by the pre-pass (hope.cu) and the kernels that rotate
// their query tiles on the fly (select_sm100.cu, attn_sm100.cu), so that both
// routes give the same bits (molayo1419.me, "Engineering details", HoPE:
// rotary embedding on the dimensions inside the pre-training window, none on
// the others).  Dimensions pair up as (i, i + d/2); pair i < npairs turns by
// pos * theta_i, theta_i = base^(-2i/d) (a double, formed once on the host).
// The angle is reduced exactly in integers: the host turns theta_i / (2 pi)
// into a 64-bit fixed-point fraction of a turn (rounded in 80-bit extended
// precision), and the fractional turn of pos * theta_i is bits 32..63 of
// pos times that fraction, two 32-bit multiplies (error below 2^-32 turn
// plus the fraction's rounding, pos * 2^-65 turn; positions below 2^31).
// That fraction, read as a signed angle in [-pi, pi), goes through the fast
// sine / cosine intrinsic (absolute error below 2^-21.4 on that interval);
// the rotation itself is fp32 with every product and sum rounded
// separately.  No double-precision arithmetic and no branch per pair.
#pragma once

#include <cuda_runtime.h>

namespace hils {

constexpr int kHopeMaxPairs = 64;

struct HopeParams {
  int npairs;  // rotated pairs (0: no rotation)
  int pos0;    // position of row 0
  unsigned long long turns[kHopeMaxPairs];  // theta_i / (2 pi) in units of 2^-64 turn
};

// the turn fractions of pairs 0 .. npairs-1 (host)
inline HopeParams hope_params(int d, int npairs, int pos0, double base);

#ifdef __CUDACC__
// 2 pi / 2^32: one unit of a 32-bit turn fraction in radians
constexpr float kHopeTurnUnit = 1.4629180792671596e-09f;

__device__ __forceinline__ void hope_sincos(unsigned long long turns, long long pos, float &sn,
                                            float &cs) {
  const uint32_t p = (uint32_t)pos;  // 0 <= pos < 2^31
  // bits 32..63 of p * turns: the fractional turn of pos * theta_i, times 2^32
  const uint32_t u = __umulhi(p, (uint32_t)turns) + p * (uint32_t)(turns >> 32);
  __sincosf((float)(int32_t)u * kHopeTurnUnit, &sn, &cs);
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
  // 1 / (2 pi) in extended precision
  const long double inv_two_pi = 0.159154943091895335768883763372514362L;
  for (int i = 0; i < npairs && i < kHopeMaxPairs; ++i) {
    const double theta = std::exp2(-(2.0 * i / d) * lb);  // at most 1
    hp.turns[i] = (unsigned long long)std::llrint(std::ldexp((long double)theta * inv_two_pi, 64));
  }
  return hp;
}
