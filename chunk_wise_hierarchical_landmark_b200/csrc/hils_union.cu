// Chunk union per group of M adjacent queries, in CSR form (molayo1419.me,
// "Hardware-efficient kernel": the chunks selected by M adjacent queries are
// loaded once as their union).  Three launches: per-group set sizes, an
// exclusive scan of the sizes, and the ascending fill.
#include "common.cuh"
#include "kernels.h"

namespace hils {

// One block per group; the group's set lives as a bitmap in shared memory.
__device__ void build_bitmap(uint32_t *bitmap, int nwords, const int32_t *sel, int head, int g,
                             int L, int C, int K, int M, uint32_t *err) {
  for (int i = threadIdx.x; i < nwords; i += blockDim.x) bitmap[i] = 0;
  __syncthreads();
  const int t0 = g * M, t1 = min(t0 + M, L);
  for (int i = threadIdx.x; i < (t1 - t0) * K; i += blockDim.x) {
    const int t = t0 + i / K;
    const int c = sel[((size_t)head * L + t) * K + (i % K)];
    if (c < 0) continue;
    if (c >= t / C) { report(err, DEV_BAD_INDEX); continue; }
    atomicOr(&bitmap[c >> 5], 1u << (c & 31));
  }
  for (int t = t0 + threadIdx.x; t < t1; t += blockDim.x) {
    const int c = t / C;
    atomicOr(&bitmap[c >> 5], 1u << (c & 31));
  }
  __syncthreads();
}

__global__ void union_count_kernel(const int32_t *__restrict__ sel, int L, int C, int K, int M,
                                   int groups_per_head, int32_t *__restrict__ counts,
                                   uint32_t *err) {
  extern __shared__ uint32_t bitmap[];
  const int nwords = ((L + C - 1) / C + 31) / 32;
  const int gid = blockIdx.x;
  build_bitmap(bitmap, nwords, sel, gid / groups_per_head, gid % groups_per_head, L, C, K, M, err);
  __shared__ int total;
  if (threadIdx.x == 0) total = 0;
  __syncthreads();
  int mine = 0;
  for (int i = threadIdx.x; i < nwords; i += blockDim.x) mine += __popc(bitmap[i]);
  atomicAdd(&total, mine);
  __syncthreads();
  if (threadIdx.x == 0) counts[gid + 1] = total;
}

// Exclusive scan of counts[1..G] into offsets[0..G] (in place), one block.
__global__ void union_scan_kernel(int32_t *__restrict__ off, int G) {
  __shared__ int carry;
  __shared__ int warp_sums[32];
  if (threadIdx.x == 0) { carry = 0; off[0] = 0; }
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int base = 0; base < G; base += blockDim.x) {
    const int i = base + threadIdx.x;
    int x = i < G ? off[i + 1] : 0;
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int s = lane < nw ? warp_sums[lane] : 0;
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
      }
      warp_sums[lane] = s;
    }
    __syncthreads();
    const int incl = x + (wid > 0 ? warp_sums[wid - 1] : 0) + carry;
    if (i < G) off[i + 1] = incl;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = incl;
    __syncthreads();
  }
}

__global__ void union_fill_kernel(const int32_t *__restrict__ sel, int L, int C, int K, int M,
                                  int groups_per_head, const int32_t *__restrict__ off,
                                  int32_t *__restrict__ u_idx, int64_t cap, uint32_t *err) {
  extern __shared__ uint32_t bitmap[];
  const int nwords = ((L + C - 1) / C + 31) / 32;
  const int gid = blockIdx.x;
  build_bitmap(bitmap, nwords, sel, gid / groups_per_head, gid % groups_per_head, L, C, K, M,
               nullptr);
  // warp 0 walks the bitmap in order and writes the ascending ids
  if (threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  int pos = off[gid];
  for (int base = 0; base < nwords; base += 32) {
    const int wi = base + lane;
    const uint32_t word = wi < nwords ? bitmap[wi] : 0u;
    const int n = __popc(word);
    int pre = n;
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, pre, o);
      if (lane >= o) pre += y;
    }
    int at = pos + pre - n;
    uint32_t x = word;
    while (x) {
      const int c = wi * 32 + __ffs(x) - 1;
      x &= x - 1;
      if (at < cap) u_idx[at] = c; else report(err, DEV_BAD_INDEX);
      ++at;
    }
    pos += __shfl_sync(0xffffffffu, pre, 31);
  }
}

cudaError_t union_csr(int B, int Hq, int L, int C, int topk, int M, const int32_t *sel,
                      int32_t *u_off, int32_t *u_idx, int64_t u_cap, uint32_t *err,
                      cudaStream_t st, int *launches) {
  const int gph = (L + M - 1) / M;
  const int G = B * Hq * gph;
  const size_t smem = (size_t)(((L + C - 1) / C + 31) / 32) * 4;
  cudaError_t e;
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(union_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(union_fill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  union_count_kernel<<<G, 256, smem, st>>>(sel, L, C, topk, M, gph, u_off, err);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  union_scan_kernel<<<1, 1024, 0, st>>>(u_off, G);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  union_fill_kernel<<<G, 256, smem, st>>>(sel, L, C, topk, M, gph, u_off, u_idx, u_cap, err);
  *launches += 3;
  return cudaGetLastError();
}

}  // namespace hils
