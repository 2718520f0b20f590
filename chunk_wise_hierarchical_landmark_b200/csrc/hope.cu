// HoPE, the hierarchical positional encoding of the pages (molayo1419.me,
// "Engineering details", HoPE): rotary position embedding on the dimensions
// whose wavelength lies inside the pre-training window, no positional
// encoding on the rest.  Dimensions pair up as (i, i + d/2); pair i turns by
// the angle t * theta_i with theta_i = base^(-2i/d), so the wavelength grows
// with i and the rotated pairs are the first n_rope_pairs (the split itself
// is the caller's: the pages give no rule).
//
// A pre-pass over q or k in HBM, bound by its bytes: one thread per
// (position, pair), pairs along threadIdx.x so a warp reads 32 consecutive
// elements of each half of a row; blockIdx.y is the (b, head) sequence, so a
// position needs no division.  The angle is formed and reduced modulo 2*pi in
// double precision (t * theta reaches ~4e6 rad at 4M tokens, where fp32
// would be off by tenths of a radian), then sincosf on the reduced angle.
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "hope.h"

namespace hils {
namespace {

constexpr int kHopeThreads = 256;
constexpr int kMaxPairs = 64;
// 2*pi as a sum of two doubles (Cody-Waite reduction)
constexpr double kTwoPiHi = 6.283185307179586;
constexpr double kTwoPiLo = 2.4492935982947064e-16;
constexpr double kInvTwoPi = 0.15915494309189535;

template <typename T>
__global__ void __launch_bounds__(kHopeThreads) hope_kernel(T *__restrict__ x, int L, int d,
                                                            int pos0, int npairs,
                                                            double log2_base) {
  __shared__ double theta[kMaxPairs];
  const int tid = threadIdx.y * blockDim.x + threadIdx.x;
  for (int i = tid; i < npairs; i += blockDim.x * blockDim.y)
    theta[i] = exp2(-(2.0 * i / d) * log2_base);
  __syncthreads();
  const int i = threadIdx.x;
  if (i >= npairs) return;
  const int half = d / 2;
  const double th = theta[i];
  T *seq = x + (size_t)blockIdx.y * L * d;
  for (int t = blockIdx.x * blockDim.y + threadIdx.y; t < L; t += gridDim.x * blockDim.y) {
    const double a = (double)(pos0 + t) * th;
    const double k = rint(a * kInvTwoPi);
    const double r = fma(-k, kTwoPiLo, fma(-k, kTwoPiHi, a));  // in [-pi, pi] up to rounding
    float sn, cs;
    sincosf((float)r, &sn, &cs);
    T *p = seq + (size_t)t * d;
    const float xi = to_f(p[i]), xj = to_f(p[i + half]);
    p[i] = from_f<T>(xi * cs - xj * sn);
    p[i + half] = from_f<T>(xi * sn + xj * cs);
  }
}

}  // namespace

cudaError_t hope_apply(void *x, bool bf16, int BH, int L, int d, int pos0, int n_rope_pairs,
                       double base, cudaStream_t st, int *launches) {
  if (n_rope_pairs <= 0) return cudaSuccess;
  const int tx = n_rope_pairs <= 32 ? 32 : 64;
  const dim3 block(tx, kHopeThreads / tx);
  const int per_block = (int)block.y;
  const int want = std::max(1, 4096 / BH);  // enough CTAs for every SM several times over
  const dim3 grid((unsigned)std::min((L + per_block - 1) / per_block, want), (unsigned)BH);
  const double lb = std::log2(base);
  if (bf16)
    hope_kernel<__nv_bfloat16><<<grid, block, 0, st>>>(static_cast<__nv_bfloat16 *>(x), L, d,
                                                       pos0, n_rope_pairs, lb);
  else
    hope_kernel<float><<<grid, block, 0, st>>>(static_cast<float *>(x), L, d, pos0,
                                               n_rope_pairs, lb);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace hils
