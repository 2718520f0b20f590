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
// (j, y) of a (r, Ty) block owns rank j for the positions y, y + Ty, ...
// (PER of them); its accumulators are independent chains, interleaved over i.
// The next slice of h and w_down is loaded into registers while the current
// one is multiplied.
template <typename T, int PER>
__global__ void __launch_bounds__(kZThreads) qcal_z_kernel(const T *__restrict__ h,
                                                          const T *__restrict__ w_down,
                                                          float *__restrict__ z, int L, int D,
                                                          int r) {
  __shared__ float hs[kPos][kDChunk + 1];
  __shared__ float ws[kMaxQcalRank][kDChunk + 1];
  constexpr int kHPer = kPos * kDChunk / kZThreads;            // h values a thread stages
  constexpr int kWPer = kMaxQcalRank * kDChunk / kZThreads;    // w values at most
  const int b = blockIdx.y, t0 = blockIdx.x * kPos;
  const int nt = blockDim.x;
  const int Ty = nt / r;  // position lanes
  const int j = threadIdx.x % r, y = threadIdx.x / r;
  float hreg[kHPer], wreg[kWPer];
  auto fetch = [&](int i0) {
    const int n = min(kDChunk, D - i0);
#pragma unroll
    for (int u = 0; u < kHPer; ++u) {
      const int e = threadIdx.x + u * nt;
      const int tt = e / kDChunk, ii = e % kDChunk;
      const int t = t0 + tt;
      hreg[u] = (e < kPos * kDChunk && t < L && ii < n)
                    ? ld_f(h + ((size_t)b * L + t) * D + i0 + ii) : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < kWPer; ++u) {
      const int e = threadIdx.x + u * nt;
      const int jj = e / kDChunk, ii = e % kDChunk;
      wreg[u] = (jj < r && ii < n) ? ld_f(w_down + (size_t)jj * D + i0 + ii) : 0.0f;
    }
  };
  float acc[PER];
#pragma unroll
  for (int u = 0; u < PER; ++u) acc[u] = 0.0f;
  fetch(0);
  for (int i0 = 0; i0 < D; i0 += kDChunk) {
    const int n = min(kDChunk, D - i0);
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kHPer; ++u) {
      const int e = threadIdx.x + u * nt;
      if (e < kPos * kDChunk) hs[e / kDChunk][e % kDChunk] = hreg[u];
    }
#pragma unroll
    for (int u = 0; u < kWPer; ++u) {
      const int e = threadIdx.x + u * nt;
      if (e / kDChunk < r) ws[e / kDChunk][e % kDChunk] = wreg[u];
    }
    __syncthreads();
    if (i0 + kDChunk < D) fetch(i0 + kDChunk);
    for (int ii = 0; ii < n; ++ii) {
      const float wv = ws[j][ii];
#pragma unroll
      for (int u = 0; u < PER; ++u) {
        const int tt = y + u * Ty;
        if (tt < kPos) acc[u] = __fadd_rn(acc[u], __fmul_rn(wv, hs[tt][ii]));
      }
    }
  }
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int tt = y + u * Ty;
    const int t = t0 + tt;
    if (tt < kPos && t < L) z[((size_t)b * L + t) * r + j] = acc[u];
  }
}

// q_cal[b, hq, t, e] = round(fl(q + sum_j fl(w_up[hq, e, j] * z[b, t, j]))), j ascending;
// RB = r rounded up to a power of two (entries past r are zero and skipped)
template <typename T, int RB>
__global__ void qcal_query_kernel(const T *__restrict__ q, const T *__restrict__ w_up,
                                  const float *__restrict__ z, T *__restrict__ q_cal, int Hq,
                                  int L, int d, int r) {
  __shared__ float zs[kPos][RB + 1];
  const int bh = blockIdx.y, b = bh / Hq, hq = bh % Hq;
  const int t0 = blockIdx.x * kPos;
  const int e = threadIdx.x;  // head dimension
  for (int i = threadIdx.x; i < kPos * r; i += blockDim.x) {
    const int tt = i / r, jj = i % r;
    const int t = t0 + tt;
    zs[tt][jj] = t < L ? z[((size_t)b * L + t) * r + jj] : 0.0f;
  }
  float wu[RB];
#pragma unroll
  for (int jj = 0; jj < RB; ++jj)
    wu[jj] = jj < r ? ld_f(w_up + ((size_t)hq * d + e) * r + jj) : 0.0f;
  __syncthreads();
  const int tn = min(kPos, L - t0);
  for (int tt = 0; tt < tn; ++tt) {
    float a = 0.0f;
    if (r == RB) {
#pragma unroll
      for (int jj = 0; jj < RB; ++jj) a = __fadd_rn(a, __fmul_rn(wu[jj], zs[tt][jj]));
    } else {
#pragma unroll
      for (int jj = 0; jj < RB; ++jj)
        if (jj < r) a = __fadd_rn(a, __fmul_rn(wu[jj], zs[tt][jj]));
    }
    const size_t off = ((size_t)bh * L + t0 + tt) * d + e;
    q_cal[off] = from_f<T>(__fadd_rn(ld_f(q + off), a));
  }
}

template <typename T>
cudaError_t qcal_launch(int B, int Hq, int L, int d, int D, int r, const void *q, const void *h,
                        const void *w_down, const void *w_up, void *q_cal, float *z,
                        cudaStream_t st) {
  const dim3 gz((L + kPos - 1) / kPos, B), gq((L + kPos - 1) / kPos, B * Hq);
  const int zthreads = (kZThreads / r) * r;  // a whole number of position lanes
  const int ty = zthreads / r;
  const int per = (kPos + ty - 1) / ty;     // positions per thread
  const T *hh = static_cast<const T *>(h), *wd = static_cast<const T *>(w_down);
#define HILS_QZ(PER) qcal_z_kernel<T, PER><<<gz, zthreads, 0, st>>>(hh, wd, z, L, D, r)
  if (per <= 1) HILS_QZ(1);
  else if (per <= 2) HILS_QZ(2);
  else if (per <= 4) HILS_QZ(4);
  else if (per <= 8) HILS_QZ(8);
  else HILS_QZ(16);
#undef HILS_QZ
  const T *qq = static_cast<const T *>(q), *wu = static_cast<const T *>(w_up);
  T *qc = static_cast<T *>(q_cal);
#define HILS_QQ(RB) qcal_query_kernel<T, RB><<<gq, d, 0, st>>>(qq, wu, z, qc, Hq, L, d, r)
  if (r <= 8) HILS_QQ(8);
  else if (r <= 16) HILS_QQ(16);
  else if (r <= 32) HILS_QQ(32);
  else HILS_QQ(64);
#undef HILS_QQ
  return cudaGetLastError();
}

}  // namespace

cudaError_t qcal_query(bool bf16, int B, int Hq, int L, int d, int D, int r, const void *q,
                       const void *h, const void *w_down, const void *w_up, void *q_cal,
                       float *z, cudaStream_t st, int *launches) {
  *launches += 2;
  return bf16 ? qcal_launch<__nv_bfloat16>(B, Hq, L, d, D, r, q, h, w_down, w_up, q_cal, z, st)
              : qcal_launch<float>(B, Hq, L, d, D, r, q, h, w_down, w_up, q_cal, z, st);
}

}  // namespace hils
