// Q-Cal scoring query (molayo1419.me, "Engineering details", Q-Cal): the
// chunk scores use q_t + W_up[hq] (W_down h_t), a low-rank learnable offset
// of the query formed from the token's hidden state h_t; attention inside the
// chunks keeps q.  Two small kernels form the calibrated query before the
// scoring kernel runs:
//   qcal_z_kernel     z[b, t, :] = W_down h[b, t, :]       (one per position,
//                     shared by every head), grid (ceil(L/64), B)
//   qcal_query_kernel q_cal = q + W_up[hq] z, rounded to the query's dtype,
//                     grid (ceil(L/64), B*Hq), one thread per head dimension
// Arithmetic (the pages give no precision; the query's own is taken): fp32,
// every product and partial sum rounded separately (__fmul_rn / __fadd_rn, no
// fused multiply-add), sums in a fixed order (over D ascending, then over r
// ascending), bf16 queries rounded to nearest even at the end.  The scoring
// pass then sees exactly the query this arithmetic defines.
#include <cuda_bf16.h>

#include "common.cuh"
#include "qcal.h"

namespace hils {
namespace {

constexpr int kPos = 64;      // positions per CTA
constexpr int kDChunk = 64;   // hidden dimensions staged per step
constexpr int kZThreads = 256;

template <typename T>
__device__ __forceinline__ float ld_f(const T *p);
template <>
__device__ __forceinline__ float ld_f<float>(const float *p) { return *p; }
template <>
__device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16 *p) {
  return __bfloat162float(*p);
}

// z[b, t, j] = sum_i fl(w_down[j, i] * h[b, t, i]), i ascending.  Thread
// (j, y) of a (r, T) block owns rank j for the positions y, y + T, ...; its
// accumulators are independent chains, interleaved over i.
template <typename T>
__global__ void __launch_bounds__(kZThreads) qcal_z_kernel(const T *__restrict__ h,
                                                          const T *__restrict__ w_down,
                                                          float *__restrict__ z, int L, int D,
                                                          int r) {
  __shared__ float hs[kPos][kDChunk + 1];
  __shared__ float ws[kMaxQcalRank][kDChunk + 1];
  const int b = blockIdx.y, t0 = blockIdx.x * kPos;
  const int Ty = blockDim.x / r;                 // position lanes
  const int j = threadIdx.x % r, y = threadIdx.x / r;
  const bool active = y < Ty;
  constexpr int kPer = kPos / (kZThreads / kMaxQcalRank);  // positions per thread at most
  float acc[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) acc[u] = 0.0f;
  for (int i0 = 0; i0 < D; i0 += kDChunk) {
    const int n = min(kDChunk, D - i0);
    __syncthreads();
    for (int e = threadIdx.x; e < kPos * kDChunk; e += blockDim.x) {
      const int tt = e / kDChunk, ii = e % kDChunk;
      const int t = t0 + tt;
      hs[tt][ii] = (t < L && ii < n) ? ld_f(h + ((size_t)b * L + t) * D + i0 + ii) : 0.0f;
    }
    for (int e = threadIdx.x; e < r * kDChunk; e += blockDim.x) {
      const int jj = e / kDChunk, ii = e % kDChunk;
      ws[jj][ii] = ii < n ? ld_f(w_down + (size_t)jj * D + i0 + ii) : 0.0f;
    }
    __syncthreads();
    if (active) {
      for (int ii = 0; ii < n; ++ii) {
        const float wv = ws[j][ii];
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
          const int tt = y + u * Ty;
          if (tt < kPos) acc[u] = __fadd_rn(acc[u], __fmul_rn(wv, hs[tt][ii]));
        }
      }
    }
  }
  if (active) {
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int tt = y + u * Ty;
      const int t = t0 + tt;
      if (tt < kPos && t < L) z[((size_t)b * L + t) * r + j] = acc[u];
    }
  }
}

// q_cal[b, hq, t, e] = round(fl(q + sum_j fl(w_up[hq, e, j] * z[b, t, j]))), j ascending
template <typename T>
__global__ void qcal_query_kernel(const T *__restrict__ q, const T *__restrict__ w_up,
                                  const float *__restrict__ z, T *__restrict__ q_cal, int Hq,
                                  int L, int d, int r) {
  __shared__ float zs[kPos][kMaxQcalRank + 1];
  const int bh = blockIdx.y, b = bh / Hq, hq = bh % Hq;
  const int t0 = blockIdx.x * kPos;
  const int e = threadIdx.x;  // head dimension
  for (int i = threadIdx.x; i < kPos * r; i += blockDim.x) {
    const int tt = i / r, j = i % r;
    const int t = t0 + tt;
    zs[tt][j] = t < L ? z[((size_t)b * L + t) * r + j] : 0.0f;
  }
  float wu[kMaxQcalRank];
#pragma unroll
  for (int j = 0; j < kMaxQcalRank; ++j)
    wu[j] = j < r ? ld_f(w_up + ((size_t)hq * d + e) * r + j) : 0.0f;
  __syncthreads();
  const int tn = min(kPos, L - t0);
  for (int tt = 0; tt < tn; ++tt) {
    float a = 0.0f;
#pragma unroll
    for (int j = 0; j < kMaxQcalRank; ++j)
      if (j < r) a = __fadd_rn(a, __fmul_rn(wu[j], zs[tt][j]));
    const size_t off = ((size_t)bh * L + t0 + tt) * d + e;
    q_cal[off] = from_f<T>(__fadd_rn(ld_f(q + off), a));
  }
}

}  // namespace

cudaError_t qcal_query(bool bf16, int B, int Hq, int L, int d, int D, int r, const void *q,
                       const void *h, const void *w_down, const void *w_up, void *q_cal,
                       float *z, cudaStream_t st, int *launches) {
  const dim3 gz((L + kPos - 1) / kPos, B), gq((L + kPos - 1) / kPos, B * Hq);
  const int zthreads = (kZThreads / r) * r;  // a whole number of position lanes
  if (bf16) {
    qcal_z_kernel<__nv_bfloat16><<<gz, zthreads, 0, st>>>(
        (const __nv_bfloat16 *)h, (const __nv_bfloat16 *)w_down, z, L, D, r);
    qcal_query_kernel<__nv_bfloat16><<<gq, d, 0, st>>>(
        (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)w_up, z, (__nv_bfloat16 *)q_cal, Hq, L, d, r);
  } else {
    qcal_z_kernel<float><<<gz, zthreads, 0, st>>>((const float *)h, (const float *)w_down, z, L,
                                                   D, r);
    qcal_query_kernel<float><<<gq, d, 0, st>>>((const float *)q, (const float *)w_up, z,
                                               (float *)q_cal, Hq, L, d, r);
  }
  *launches += 2;
  return cudaGetLastError();
}

}  // namespace hils
