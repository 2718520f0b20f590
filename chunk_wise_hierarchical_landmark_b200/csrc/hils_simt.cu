// CUDA-core (SIMT) kernels of the HiLS forward pass, used for fp32 inputs
// (tensor cores have no exact fp32 path) and for the decode step's row.
//
//   select_simt : landmark logits s_c = scale * <q_t, lmk_c> for completed
//                 chunks c < floor(t/C), their log-sum-exp, and a top-k by
//                 (s desc, c asc) -- model card "HiLS-Attention", section
//                 "What HiLS-Attention is"; molayo1419.me, "Core idea" step 1.
//   attn_simt   : attention inside the selected chunks and the causal own
//                 chunk, fused by the chunk logits -- molayo1419.me, "Core
//                 idea" step 2; aiweekly.co, mechanism paragraph.  The tile's
//                 chunk union is built in shared memory and each chunk's K/V
//                 is staged once for all rows of the tile (molayo1419.me,
//                 "Hardware-efficient kernel").
#include "common.cuh"
#include "kernels.h"

namespace hils {

// fp32 inputs take the accurate expf/logf (the fp32 path is held to 1e-5);
// bf16 inputs take the fast intrinsics.
template <typename T>
__device__ __forceinline__ float ex(float x) { return __expf(x); }
template <>
__device__ __forceinline__ float ex<float>(float x) { return expf(x); }
template <typename T>
__device__ __forceinline__ float lg(float x) { return __logf(x); }
template <>
__device__ __forceinline__ float lg<float>(float x) { return logf(x); }

// ---------------------------------------------------------------------------
// select_simt: one thread per query row, 128 rows per block.
template <typename T, int D>
__global__ void __launch_bounds__(128) select_simt_kernel(RowSpec rs, const T *__restrict__ q,
                                                          const T *__restrict__ lmk,
                                                          int32_t *__restrict__ sel,
                                                          float *__restrict__ w,
                                                          float *__restrict__ lse_lmk) {
  extern __shared__ __align__(16) unsigned char smem[];
  float *qs = reinterpret_cast<float *>(smem);   // [128][D+1]
  float *ls = qs + 128 * (D + 1);                // [32][D]
  uint64_t *keys = reinterpret_cast<uint64_t *>(ls + 32 * D);  // [topk][128]

  const int tid = threadIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / rs.Hq, hq = bh % rs.Hq, hkv = hq / (rs.Hq / rs.Hkv);
  const int r0 = blockIdx.x * 128;                // row offset within [0, t_count)
  const int nrows = min(128, rs.t_count - r0);
  const bool valid = tid < nrows;
  const int t = rs.t_first + r0 + tid;

  for (int i = tid; i < 128 * D; i += 128) {
    const int r = i / D, e = i % D;
    qs[r * (D + 1) + e] =
        r < nrows ? to_f(q[((size_t)bh * rs.t_count + r0 + r) * D + e]) : 0.0f;
  }
  const int nlmk = rs.L / rs.C;
  const int n_c = valid ? t / rs.C : 0;
  const int t_last = rs.t_first + r0 + nrows - 1;
  const int n_c_max = min(t_last / rs.C, nlmk);
  const T *lhead = lmk + (size_t)(b * rs.Hkv + hkv) * nlmk * D;

  float m = -INFINITY, l = 0.0f;
  int cnt = 0, minpos = 0;
  uint64_t minkey = 0;
  const int K = rs.topk;

  for (int c0 = 0; c0 < n_c_max; c0 += 32) {
    __syncthreads();
    for (int i = tid; i < 32 * D; i += 128) {
      const int c = c0 + i / D;
      ls[i] = c < nlmk ? to_f(lhead[(size_t)c * D + (i % D)]) : 0.0f;
    }
    __syncthreads();
    const int cend = min(32, n_c - c0);
    for (int r = 0; r < cend; ++r) {
      float acc = 0.0f;
#pragma unroll 16
      for (int e = 0; e < D; ++e) acc = fmaf(qs[tid * (D + 1) + e], ls[r * D + e], acc);
      const float s = acc * rs.scale;
      if (s > m) {
        l = l * ex<T>(m - s) + 1.0f;
        m = s;
      } else {
        l += ex<T>(s - m);
      }
      const uint64_t key = sel_key(s, c0 + r);
      if (cnt < K) {
        keys[cnt * 128 + tid] = key;
        ++cnt;
        if (cnt == K) {
          minkey = keys[tid];
          minpos = 0;
          for (int i = 1; i < K; ++i)
            if (keys[i * 128 + tid] < minkey) { minkey = keys[i * 128 + tid]; minpos = i; }
        }
      } else if (key > minkey) {
        keys[minpos * 128 + tid] = key;
        minkey = keys[tid];
        minpos = 0;
        for (int i = 1; i < K; ++i)
          if (keys[i * 128 + tid] < minkey) { minkey = keys[i * 128 + tid]; minpos = i; }
      }
    }
  }
  if (!valid) return;
  // ascending chunk order (insertion sort on the chunk id)
  for (int i = 1; i < cnt; ++i) {
    const uint64_t x = keys[i * 128 + tid];
    int j = i - 1;
    while (j >= 0 && key_chunk(keys[j * 128 + tid]) > key_chunk(x)) {
      keys[(j + 1) * 128 + tid] = keys[j * 128 + tid];
      --j;
    }
    keys[(j + 1) * 128 + tid] = x;
  }
  const size_t row = (size_t)bh * rs.t_count + r0 + tid;
  for (int i = 0; i < K; ++i) {
    const bool have = i < cnt;
    sel[row * K + i] = have ? key_chunk(keys[i * 128 + tid]) : -1;
    w[row * K + i] = have ? key_score(keys[i * 128 + tid]) : -INFINITY;
  }
  if (lse_lmk) lse_lmk[row] = n_c > 0 ? m + lg<T>(l) : -INFINITY;
}

// ---------------------------------------------------------------------------
// attn_simt: 64 rows (one chunk's worth of positions, so one own chunk) per
// block, 4 threads per row each owning D/4 of the head dimension.
template <typename T, int D>
__global__ void __launch_bounds__(256) attn_simt_kernel(RowSpec rs, const T *__restrict__ q,
                                                        const T *__restrict__ k,
                                                        const T *__restrict__ v,
                                                        const int32_t *__restrict__ sel,
                                                        const float *__restrict__ w,
                                                        T *__restrict__ out,
                                                        float *__restrict__ lse,
                                                        float *__restrict__ wfin,
                                                        uint32_t *__restrict__ err) {
  constexpr int DP = D / 4;
  constexpr int TR = 64;
  extern __shared__ __align__(16) unsigned char smem[];
  float *ks = reinterpret_cast<float *>(smem);  // [64][D]
  float *vs = ks + TR * D;                      // [64][D]
  uint32_t *bitmap = reinterpret_cast<uint32_t *>(vs + TR * D);

  const int tid = threadIdx.x, rloc = tid >> 2, part = tid & 3;
  // the four threads of a row exchange partial dot products among themselves
  const unsigned qmask = 0xFu << (tid & 28);
  const int bh = blockIdx.y;
  const int b = bh / rs.Hq, hq = bh % rs.Hq, hkv = hq / (rs.Hq / rs.Hkv);
  const int C = rs.C, K = rs.topk;
  const int p0 = (rs.t_first / TR) * TR + blockIdx.x * TR;  // first position of the tile
  const int t = p0 + rloc;
  const bool valid = t >= rs.t_first && t < rs.t_first + rs.t_count;
  const int nchunks = (rs.L + C - 1) / C;
  const int nwords = (nchunks + 31) / 32;
  const size_t row = valid ? (size_t)bh * rs.t_count + (t - rs.t_first) : 0;
  const size_t kvhead = (size_t)(b * rs.Hkv + hkv) * rs.L;

  for (int i = tid; i < nwords; i += 256) bitmap[i] = 0;
  __syncthreads();
  // union of the tile's selections (own chunk handled separately)
  for (int i = tid; i < TR * K; i += 256) {
    const int rr = i / K, tt = p0 + rr;
    if (tt < rs.t_first || tt >= rs.t_first + rs.t_count) continue;
    const int c = sel[((size_t)bh * rs.t_count + (tt - rs.t_first)) * K + (i % K)];
    if (c < 0) continue;
    if (c >= tt / C) { report(err, DEV_BAD_INDEX); continue; }
    atomicOr(&bitmap[c >> 5], 1u << (c & 31));
  }

  float qv[DP], acc[DP];
#pragma unroll
  for (int e = 0; e < DP; ++e) {
    qv[e] = valid ? to_f(q[row * D + part * DP + e]) * rs.scale : 0.0f;
    acc[e] = 0.0f;
  }
  // the row's selection: ascending ids, -1 padding at the end
  const int32_t *mysel = sel + row * K;
  const float *myw = w + row * K;
  int nsel = 0;
  float wmax = -INFINITY;
  if (valid)
    for (int i = 0; i < K; ++i) {
      const int c = mysel[i];
      if (c >= 0) { ++nsel; wmax = fmaxf(wmax, myw[i]); }
    }
  int ptr = 0;
  float Mrow = 0.0f, lse_own = 0.0f;
  const int own = p0 / C;

  auto stage = [&](int c) {
    __syncthreads();
    for (int i = tid; i < TR * D; i += 256) {
      const int j = c * C + i / D;
      const bool in = (i / D) < C && j < rs.L;
      ks[i] = in ? to_f(k[(kvhead + j) * D + (i % D)]) : 0.0f;
      vs[i] = in ? to_f(v[(kvhead + j) * D + (i % D)]) : 0.0f;
    }
    __syncthreads();
  };
  // logits x_j = scale * <q, k_j> for the keys of the staged chunk; jmax = last key
  auto logits = [&](float *x, int jmax) {
#pragma unroll
    for (int j = 0; j < TR; ++j) {
      float a = 0.0f;
#pragma unroll
      for (int e = 0; e < DP; ++e) a = fmaf(qv[e], ks[j * D + part * DP + e], a);
      a += __shfl_xor_sync(qmask, a, 1);
      a += __shfl_xor_sync(qmask, a, 2);
      x[j] = j <= jmax ? a : -INFINITY;
    }
  };

  float x[TR];
  // own chunk first: its logit (exact log mass of the causal keys) fixes the
  // row's reference maximum M = max(lse_own, max selected logit)
  stage(own);
  if (valid) {
    logits(x, t - own * C);
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < TR; ++j) m = fmaxf(m, x[j]);
    float l = 0.0f;
#pragma unroll
    for (int j = 0; j < TR; ++j) { x[j] = ex<T>(x[j] - m); l += x[j]; }
    lse_own = m + lg<T>(l);
    Mrow = fmaxf(lse_own, wmax);
    const float sc = ex<T>(lse_own - Mrow) / l;
#pragma unroll
    for (int j = 0; j < TR; ++j) {
      const float p = x[j] * sc;
#pragma unroll
      for (int e = 0; e < DP; ++e) acc[e] = fmaf(p, vs[j * D + part * DP + e], acc[e]);
    }
  }
  __syncthreads();
  if (tid == 0 && own < nchunks) bitmap[own >> 5] &= ~(1u << (own & 31));
  __syncthreads();

  for (int wi = 0; wi < nwords; ++wi) {
    uint32_t word = bitmap[wi];
    while (word) {
      const int c = wi * 32 + __ffs(word) - 1;
      word &= word - 1;
      stage(c);
      const bool mine = valid && ptr < nsel && mysel[ptr] == c;
      if (mine) {
        const float s = myw[ptr];
        ++ptr;
        logits(x, TR - 1);
        float m = -INFINITY;
#pragma unroll
        for (int j = 0; j < TR; ++j) m = fmaxf(m, x[j]);
        float l = 0.0f;
#pragma unroll
        for (int j = 0; j < TR; ++j) { x[j] = ex<T>(x[j] - m); l += x[j]; }
        const float sc = ex<T>(s - Mrow) / l;
#pragma unroll
        for (int j = 0; j < TR; ++j) {
          const float p = x[j] * sc;
#pragma unroll
          for (int e = 0; e < DP; ++e) acc[e] = fmaf(p, vs[j * D + part * DP + e], acc[e]);
        }
      }
    }
  }
  if (!valid) return;
  if (ptr != nsel) report(err, DEV_BAD_INDEX);
  float lsum = ex<T>(lse_own - Mrow);
  for (int i = 0; i < nsel; ++i) lsum += ex<T>(myw[i] - Mrow);
  const float inv = 1.0f / lsum;
#pragma unroll
  for (int e = 0; e < DP; ++e) out[row * D + part * DP + e] = from_f<T>(acc[e] * inv);
  const float lse_row = Mrow + lg<T>(lsum);
  if (part == 0) {
    lse[row] = lse_row;
    if (wfin) {
      for (int i = 0; i < K; ++i)
        wfin[row * (K + 1) + i] = i < nsel ? ex<T>(myw[i] - lse_row) : 0.0f;
      wfin[row * (K + 1) + K] = ex<T>(lse_own - lse_row);
    }
  }
}

// ---------------------------------------------------------------------------
// launchers

template <typename T, int D>
static cudaError_t launch_select(const RowSpec &rs, const void *q, const void *lmk, int32_t *sel,
                                 float *w, float *lse_lmk, cudaStream_t st) {
  const size_t smem = (size_t)128 * (D + 1) * 4 + 32 * D * 4 + (size_t)rs.topk * 128 * 8;
  auto kern = select_simt_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((rs.t_count + 127) / 128, rs.B * rs.Hq);
  kern<<<grid, 128, smem, st>>>(rs, (const T *)q, (const T *)lmk, sel, w, lse_lmk);
  return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t launch_attn(const RowSpec &rs, const void *q, const void *k, const void *v,
                               const int32_t *sel, const float *w, void *out, float *lse,
                               float *wfin, uint32_t *err, cudaStream_t st) {
  const int nchunks = (rs.L + rs.C - 1) / rs.C;
  const size_t smem = (size_t)2 * 64 * D * 4 + (size_t)((nchunks + 31) / 32) * 4;
  auto kern = attn_simt_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int tiles = (rs.t_first % 64 + rs.t_count + 63) / 64;
  dim3 grid(tiles, rs.B * rs.Hq);
  kern<<<grid, 256, smem, st>>>(rs, (const T *)q, (const T *)k, (const T *)v, sel, w, (T *)out,
                                lse, wfin, err);
  return cudaGetLastError();
}

size_t simt_attn_smem(int d, int L, int C) {
  return (size_t)2 * 64 * d * 4 + (size_t)(((L + C - 1) / C + 31) / 32) * 4;
}

cudaError_t select_simt(const RowSpec &rs, bool bf16, const void *q, const void *lmk,
                        int32_t *sel, float *w, float *lse_lmk, cudaStream_t st) {
  if (bf16)
    return rs.d == 64 ? launch_select<__nv_bfloat16, 64>(rs, q, lmk, sel, w, lse_lmk, st)
                      : launch_select<__nv_bfloat16, 128>(rs, q, lmk, sel, w, lse_lmk, st);
  return rs.d == 64 ? launch_select<float, 64>(rs, q, lmk, sel, w, lse_lmk, st)
                    : launch_select<float, 128>(rs, q, lmk, sel, w, lse_lmk, st);
}

cudaError_t attn_simt(const RowSpec &rs, bool bf16, const void *q, const void *k, const void *v,
                      const int32_t *sel, const float *w, void *out, float *lse, float *wfin,
                      uint32_t *err, cudaStream_t st) {
  if (bf16)
    return rs.d == 64
               ? launch_attn<__nv_bfloat16, 64>(rs, q, k, v, sel, w, out, lse, wfin, err, st)
               : launch_attn<__nv_bfloat16, 128>(rs, q, k, v, sel, w, out, lse, wfin, err, st);
  return rs.d == 64 ? launch_attn<float, 64>(rs, q, k, v, sel, w, out, lse, wfin, err, st)
                    : launch_attn<float, 128>(rs, q, k, v, sel, w, out, lse, wfin, err, st);
}

}  // namespace hils
