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
// position needs no division.  The angle and the rotation are those of
// hope.cuh, shared with the kernels that rotate queries on the fly.
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "hope.cuh"
#include "hope.h"

namespace hils {
namespace {

constexpr int kHopeThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kHopeThreads) hope_kernel(T *__restrict__ x, int L, int d,
                                                            const HopeParams hp) {
  const int i = threadIdx.x;
  if (i >= hp.npairs) return;
  const int half = d / 2;
  const unsigned long long th = hp.turns[i];
  T *seq = x + (size_t)blockIdx.y * L * d;
  for (int t = blockIdx.x * blockDim.y + threadIdx.y; t < L; t += gridDim.x * blockDim.y) {
    float sn, cs;
    hope_sincos(th, (long long)hp.pos0 + t, sn, cs);
    T *p = seq + (size_t)t * d;
    float yi, yj;
    hope_rotate(to_f(p[i]), to_f(p[i + half]), sn, cs, yi, yj);
    p[i] = from_f<T>(yi);
    p[i + half] = from_f<T>(yj);
  }
}

}  // namespace

cudaError_t hope_apply(void *x, bool bf16, int BH, int L, int d, int pos0, int n_rope_pairs,
                       double base, cudaStream_t st, int *launches) {
  if (n_rope_pairs <= 0) return cudaSuccess;
  const HopeParams hp = hope_params(d, n_rope_pairs, pos0, base);
  const int tx = n_rope_pairs <= 32 ? 32 : 64;
  const dim3 block(tx, kHopeThreads / tx);
  const int per_block = (int)block.y;
  const int want = std::max(1, 4096 / BH);  // enough CTAs for every SM several times over
  const dim3 grid((unsigned)std::min((L + per_block - 1) / per_block, want), (unsigned)BH);
  if (bf16)
    hope_kernel<__nv_bfloat16><<<grid, block, 0, st>>>(static_cast<__nv_bfloat16 *>(x), L, d, hp);
  else
    hope_kernel<float><<<grid, block, 0, st>>>(static_cast<float *>(x), L, d, hp);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace hils
