// Backward pass of the HiLS forward (aiweekly.co, the paragraph on the
// mechanism: the chunk outputs are fused by the chunk retrieval scores, so
// the loss reaches those scores; molayo1419.me, "Core idea": the landmark keys
// take part in the forward pass and are trained by it).  The top-k choice is
// a discrete decision and carries no gradient; the forward's selection
// (sel_idx), its landmark logits (chunk_w) and its lse are inputs.
//
// Per row t and attended chunk c (its selected chunks, slots 0..k-1, and its
// own chunk, slot k), with p the softmax inside the chunk and w the fusion
// weights (out = sum_c w_c sum_j p_cj v_j):
//   dP_j = <dO, v_j>,  g_c = sum_j p_cj dP_j = <dO, O_c>,  D = sum_c w_c g_c
//   ds_c = w_c (g_c - D + dlse)                      (the chunk's fusion logit)
//   dx_j = w_c p_cj (dP_j - g_c) [+ p_own,j ds_own]  (the own chunk's logit is
//                                                     its log-sum-exp)
//   dq_t  = scale (sum_cj dx_j k_j + sum_{c selected} ds_c lmk_c)
//   dk_j += scale dx_j q_t,  dv_j += w_c p_cj dO_t,  dlmk_c += scale ds_c q_t
// Three stages, all on the CUDA cores with fp32 arithmetic (bf16 inputs widen
// exactly, or enter a mixed-precision FMA whose products are exact):
//   bwd_rows_kernel   one warp per row (eight lanes per key, four keys per
//                     step), one pass over its chunks: per-chunk softmax
//                     recomputed from q and the chunk's keys, g_c, w_c, and
//                     dq with the D-dependent part factored out; then D and
//                     the per-(row, slot) records (lse_c, w_c, g_c, ds_c).
//   transposed selection: per (b, kv head, chunk) the (row, slot) pairs that
//                     select it (counted by the row pass, exclusive scan,
//                     fill; the order inside a chunk's list follows the atomic
//                     fill).
//   bwd_chunks_kernel one CTA per (b, kv head, chunk): a thread per (keys,
//                     quarter of the head dimension; two keys at d = 64),
//                     that quarter of its keys' K and V rows in registers,
//                     accumulating dk and dv over the rows that attend the
//                     chunk (its own rows, causally, and the rows that
//                     selected it; staged in shared memory in batches), dlmk
//                     over the selecting rows.
#include <cuda_bf16.h>

#include <type_traits>

#include "backward.h"
#include "common.cuh"

namespace hils {
namespace {

constexpr int kC = 64;
constexpr int kRowWarps = 8;       // rows per CTA of the row pass
constexpr int kRowBatch = 32;      // rows staged together in the chunk pass

// Eight consecutive elements of a row (16-byte aligned) widened to fp32.
template <typename T>
__device__ __forceinline__ void ld8(const T *p, float (&f)[8]);
template <>
__device__ __forceinline__ void ld8<__nv_bfloat16>(const __nv_bfloat16 *p, float (&f)[8]) {
  const uint4 w = *reinterpret_cast<const uint4 *>(p);
  const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    f[2 * u] = __uint_as_float(ww[u] << 16);
    f[2 * u + 1] = __uint_as_float(ww[u] & 0xFFFF0000u);
  }
}
template <>
__device__ __forceinline__ void ld8<float>(const float *p, float (&f)[8]) {
  const float4 a = *reinterpret_cast<const float4 *>(p), b = *reinterpret_cast<const float4 *>(p + 4);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

// n consecutive elements (a multiple of 8, 16-byte aligned) widened to fp32
template <typename T, int N>
__device__ __forceinline__ void ld_vec(const T *p, float (&f)[N]) {
#pragma unroll
  for (int u = 0; u < N; u += 8) {
    float g[8];
    ld8<T>(p + u, g);
#pragma unroll
    for (int i = 0; i < 8; ++i) f[u + i] = g[i];
  }
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// acc += a * x over a lane's dimensions, as fp32 pairs
template <int N>
__device__ __forceinline__ void axpy2(float a, const float (&x)[N], float (&acc)[N]) {
  const float2 a2 = make_float2(a, a);
#pragma unroll
  for (int u = 0; u < N; u += 2) {
    const float2 t = __ffma2_rn(a2, make_float2(x[u], x[u + 1]), make_float2(acc[u], acc[u + 1]));
    acc[u] = t.x;
    acc[u + 1] = t.y;
  }
}

// <x, y> over a lane's dimensions, fp32 pairs
template <int N>
__device__ __forceinline__ float dot2(const float (&x)[N], const float (&y)[N]) {
  float2 a = make_float2(0.0f, 0.0f);
#pragma unroll
  for (int u = 0; u < N; u += 2)
    a = __ffma2_rn(make_float2(x[u], x[u + 1]), make_float2(y[u], y[u + 1]), a);
  return a.x + a.y;
}

// e += a.lo * b.lo, o += a.hi * b.hi for two packed bf16 pairs: the mixed-
// precision FMA (bf16 operands, fp32 addend and result) rounds once, and a
// product of two bf16 values is exact in fp32, so this equals widening both
// operands and an fp32 FMA, without the widening instructions.
__device__ __forceinline__ void fma_bf16x2(uint32_t a, uint32_t b, float &e, float &o) {
  asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
      "mov.b32 {al, ah}, %2;\n\t"
      "mov.b32 {bl, bh}, %3;\n\t"
      "fma.rn.f32.bf16 %0, al, bl, %0;\n\t"
      "fma.rn.f32.bf16 %1, ah, bh, %1;\n\t}"
      : "+f"(e), "+f"(o)
      : "r"(a), "r"(b));
}

// <row, x> over a lane's N dimensions (16-byte aligned bf16 row, x as packed
// bf16 pairs): even and odd dimensions summed apart and added at the end, the
// order dot2 uses
template <int N>
__device__ __forceinline__ float dot_bf16(const __nv_bfloat16 *row, const uint32_t (&x)[N / 2]) {
  float e = 0.0f, o = 0.0f;
#pragma unroll
  for (int u = 0; u < N; u += 8) {
    const uint4 w = *reinterpret_cast<const uint4 *>(row + u);
    fma_bf16x2(w.x, x[u / 2], e, o);
    fma_bf16x2(w.y, x[u / 2 + 1], e, o);
    fma_bf16x2(w.z, x[u / 2 + 2], e, o);
    fma_bf16x2(w.w, x[u / 2 + 3], e, o);
  }
  return e + o;
}

// A warp per row.  Lane layout: eight lanes per key (sub = lane & 7 holds the
// head dimensions [sub * DL, sub * DL + DL)), four keys per step (grp =
// lane >> 3 takes key 4 i + grp at step i), so a 16-byte load of the warp
// covers four whole key rows and a dot product needs three shuffle levels.
template <typename T, int D>
__global__ void __launch_bounds__(kRowWarps * 32, D == 64 ? 3 : 2)  // resident CTAs: a latency-bound loop
    bwd_rows_kernel(BwdSpec bs, const T *__restrict__ q, const T *__restrict__ k,
                    const T *__restrict__ v, const T *__restrict__ lmk,
                    const int32_t *__restrict__ sel, const float *__restrict__ chunk_w,
                    const float *__restrict__ lse, const T *__restrict__ dout,
                    const float *__restrict__ dlse, float4 *__restrict__ rec,
                    float *__restrict__ dq, uint32_t *__restrict__ cnt,
                    uint32_t *__restrict__ err) {
  constexpr int DL = D / 8;  // dimensions per lane
  const int lane = threadIdx.x & 31, sub = lane & 7, grp = lane >> 3;
  const int wi = threadIdx.x >> 5;
  const long long row = (long long)blockIdx.x * kRowWarps + wi;
  if (row >= (long long)bs.B * bs.Hq * bs.L) return;
  const int L = bs.L, K = bs.topk;
  const int bh = (int)(row / L), t = (int)(row % L);
  const int b = bh / bs.Hq, hq = bh % bs.Hq, hkv = hq / (bs.Hq / bs.Hkv);
  const int own = t / kC;
  const size_t kv0 = ((size_t)b * bs.Hkv + hkv) * L;  // first key row of the KV head
  // per warp: (x, dP) and then (p, p dP) of the chunk's keys
  __shared__ float2 xd_s[kRowWarps][kC], pd_s[kRowWarps][kC];
  float2 *xd = xd_s[wi], *pp = pd_s[wi];
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  float qv[DL], dov[DL];
  uint32_t qp[DL / 2], dop[DL / 2];  // bf16: the lane's q and dO as packed pairs
  if constexpr (kBf16) {
#pragma unroll
    for (int u = 0; u < DL; u += 8) {
      const uint4 a = *reinterpret_cast<const uint4 *>(q + (size_t)row * D + sub * DL + u);
      const uint4 c = *reinterpret_cast<const uint4 *>(dout + (size_t)row * D + sub * DL + u);
      qp[u / 2] = a.x; qp[u / 2 + 1] = a.y; qp[u / 2 + 2] = a.z; qp[u / 2 + 3] = a.w;
      dop[u / 2] = c.x; dop[u / 2 + 1] = c.y; dop[u / 2 + 2] = c.z; dop[u / 2 + 3] = c.w;
    }
  } else {
    ld_vec<T, DL>(q + (size_t)row * D + sub * DL, qv);
    ld_vec<T, DL>(dout + (size_t)row * D + sub * DL, dov);
  }
  const float lse_t = lse[row];
  const float dl = dlse ? dlse[row] : 0.0f;
  const int32_t *srow = sel + (size_t)row * K;
  const float *wrow = chunk_w + (size_t)row * K;
  float4 *rrow = rec + (size_t)row * (K + 1);

  // One pass over the attended chunks.  w_c = exp(s_c - lse) is known up
  // front, so dq splits into terms that need no D = sum_c w_c g_c and one
  // that is D times a vector:
  //   dq / scale = sum_c w_c (A_c - g_c B_c)              A_c = sum_j p_cj dP_cj k_j
  //              + sum_sel w_c (g_c + dlse) lmk_c          B_c = sum_j p_cj k_j
  //              + w_own (g_own + dlse) B_own
  //              - D (sum_sel w_c lmk_c + w_own B_own)
  // (the ds_c = w_c (g_c - D + dlse) terms and the own chunk's p ds_own term
  // regrouped); ds_c goes into the records afterwards.  Every term is linear
  // in A_c and B_c, so each key group accumulates its own keys' share and the
  // four groups are summed once, at the end.
  float acc[DL], accd[DL];
#pragma unroll
  for (int u = 0; u < DL; ++u) acc[u] = accd[u] = 0.0f;
  float Dsum = 0.0f;
  const float g0 = grp == 0 ? 1.0f : 0.0f;  // the landmark terms enter once
  for (int slot = 0; slot <= K; ++slot) {
    int c;
    float s_sel = 0.0f;
    if (slot < K) {
      c = srow[slot];
      if (c < 0) continue;
      if (c >= own) {
        report(err, DEV_BAD_INDEX);
        continue;
      }
      s_sel = wrow[slot];
    } else {
      c = own;
    }
    const int nkeys = slot < K ? kC : t - own * kC + 1;
    const int nsteps = (nkeys + 3) >> 2;
    const T *kc = k + (kv0 + (size_t)c * kC) * D + sub * DL;
    const T *vc = v + (kv0 + (size_t)c * kC) * D + sub * DL;
    __syncwarp();  // the previous chunk's reads of xd and pp are done
#pragma unroll 8
    for (int i = 0; i < nsteps; ++i) {
      const int jj = 4 * i + grp, j = min(jj, nkeys - 1);
      float a, d;
      if constexpr (kBf16) {
        a = dot_bf16<DL>(kc + (size_t)j * D, qp);
        d = dot_bf16<DL>(vc + (size_t)j * D, dop);
      } else {
        float fk[DL], fv[DL];
        ld_vec<T, DL>(kc + (size_t)j * D, fk);
        ld_vec<T, DL>(vc + (size_t)j * D, fv);
        a = dot2<DL>(fk, qv);
        d = dot2<DL>(fv, dov);
      }
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, o);
        d += __shfl_xor_sync(0xffffffffu, d, o);
      }
      if (sub == 0) xd[jj] = make_float2(a * bs.scale, d);
    }
    __syncwarp();
    // softmax over keys lane and lane + 32
    const bool in0 = lane < nkeys, in1 = lane + 32 < nkeys;
    const float2 r0 = in0 ? xd[lane] : make_float2(0.0f, 0.0f);
    const float2 r1 = in1 ? xd[lane + 32] : make_float2(0.0f, 0.0f);
    const float m = warp_max(fmaxf(in0 ? r0.x : -INFINITY, in1 ? r1.x : -INFINITY));
    const float e0 = in0 ? __expf(r0.x - m) : 0.0f, e1 = in1 ? __expf(r1.x - m) : 0.0f;
    const float l = warp_sum(e0 + e1);
    const float lc = m + __logf(l);
    const float g = warp_sum(e0 * r0.y + e1 * r1.y) / l;
    const float s = slot < K ? s_sel : lc;
    const float w = __expf(s - lse_t);
    Dsum += w * g;
    if (lane == 0) rrow[slot] = make_float4(lc, w, g, 0.0f);
    const float p0 = e0 / l, p1 = e1 / l;
    pp[lane] = make_float2(p0, p0 * r0.y);
    pp[lane + 32] = make_float2(p1, p1 * r1.y);
    __syncwarp();
    // the group's share of A_c and B_c (keys past nkeys have p = 0)
    float av[DL], bv[DL];
#pragma unroll
    for (int u = 0; u < DL; ++u) av[u] = bv[u] = 0.0f;
#pragma unroll 8
    for (int i = 0; i < nsteps; ++i) {
      const int jj = 4 * i + grp, j = min(jj, nkeys - 1);
      const float2 pj = pp[jj];
      float fk[DL];
      ld_vec<T, DL>(kc + (size_t)j * D, fk);
      axpy2<DL>(pj.y, fk, av);
      axpy2<DL>(pj.x, fk, bv);
    }
    const float wg = w * (g + dl);
#pragma unroll
    for (int u = 0; u < DL; ++u) av[u] -= g * bv[u];
    axpy2<DL>(w, av, acc);
    if (slot < K) {
      float f[DL];
      ld_vec<T, DL>(lmk + (((size_t)b * bs.Hkv + hkv) * bs.nlmk + c) * D + sub * DL, f);
      axpy2<DL>(wg * g0, f, acc);
      axpy2<DL>(w * g0, f, accd);
    } else {
      axpy2<DL>(wg, bv, acc);
      axpy2<DL>(w, bv, accd);
    }
  }
  // sum the four key groups; group 0 writes the lane's dimensions of dq
#pragma unroll
  for (int u = 0; u < DL; ++u) {
    acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], 8);
    acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], 16);
    accd[u] += __shfl_xor_sync(0xffffffffu, accd[u], 8);
    accd[u] += __shfl_xor_sync(0xffffffffu, accd[u], 16);
  }
  if (grp == 0) {
    float *dqr = dq + (size_t)row * D + sub * DL;
#pragma unroll
    for (int u = 0; u < DL; u += 4)
      *reinterpret_cast<float4 *>(dqr + u) =
          make_float4((acc[u] - Dsum * accd[u]) * bs.scale, (acc[u + 1] - Dsum * accd[u + 1]) * bs.scale,
                      (acc[u + 2] - Dsum * accd[u + 2]) * bs.scale, (acc[u + 3] - Dsum * accd[u + 3]) * bs.scale);
  }
  // ds_c = w_c (g_c - D + dlse) into the records of the attended slots, and
  // the count of the (row, slot) pairs that select each chunk (the
  // transposed selection's first step)
  __syncwarp();
  for (int slot = lane; slot <= K; slot += 32) {
    if (slot < K) {
      const int c = srow[slot];
      if (c < 0 || c >= own) continue;
      atomicAdd(&cnt[((size_t)b * bs.Hkv + hkv) * bs.nch + c], 1u);
    }
    float4 r4 = rrow[slot];
    r4.w = r4.y * (r4.z - Dsum + dl);
    rrow[slot] = r4;
  }
}

// the (row, slot) pairs that select each (b, kv head, chunk): counted by
// the row pass ...
// ... exclusive scan (one CTA; the counts become the fill cursors, zeroed) ...
__global__ void __launch_bounds__(1024) bwd_scan_kernel(uint32_t *__restrict__ cnt,
                                                        uint32_t *__restrict__ off, int n) {
  __shared__ uint32_t wsum[32];
  __shared__ uint32_t carry_s;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) carry_s = 0;
  __syncthreads();
  for (int base = 0; base < n; base += 1024) {
    const int i = base + tid;
    const uint32_t c = i < n ? cnt[i] : 0u;
    uint32_t x = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    if (warp == 0) {
      uint32_t s = wsum[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
      }
      wsum[lane] = s;
    }
    __syncthreads();
    const uint32_t carry = carry_s;
    const uint32_t excl = carry + (warp > 0 ? wsum[warp - 1] : 0u) + x - c;
    if (i < n) {
      off[i] = excl;
      cnt[i] = 0u;
    }
    __syncthreads();
    if (tid == 1023) carry_s = excl + c;
    __syncthreads();
  }
  if (tid == 0) off[n] = carry_s;
}

// ... and fill
__global__ void bwd_fill_kernel(BwdSpec bs, const int32_t *__restrict__ sel,
                                const uint32_t *__restrict__ off, uint32_t *__restrict__ cur,
                                int32_t *__restrict__ ent_row, uint8_t *__restrict__ ent_slot) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long n = (long long)bs.B * bs.Hq * bs.L * bs.topk;
  if (i >= n) return;
  const int c = sel[i];
  const long long row = i / bs.topk;
  const int t = (int)(row % bs.L), bh = (int)(row / bs.L);
  if (c < 0 || c >= t / kC) return;
  const int b = bh / bs.Hq, hkv = (bh % bs.Hq) / (bs.Hq / bs.Hkv);
  const size_t seg = ((size_t)b * bs.Hkv + hkv) * bs.nch + c;
  const uint32_t pos = off[seg] + atomicAdd(&cur[seg], 1u);
  ent_row[pos] = (int32_t)row;
  ent_slot[pos] = (uint8_t)(i % bs.topk);
}

// Keys per thread of the chunk pass: two at d = 64 (each staged q / dO value
// read from shared memory then feeds two keys), one at d = 128 (registers).
template <int D>
struct ChunkCfg {
  static constexpr int kKeys = D == 64 ? 2 : 1;
  static constexpr int kThreads = kC * 4 / kKeys;
  static constexpr int kMinBlocks = D == 64 ? 3 : 1;
};

template <typename T, int D>
__global__ void __launch_bounds__(ChunkCfg<D>::kThreads, ChunkCfg<D>::kMinBlocks)
    bwd_chunks_kernel(BwdSpec bs, const T *__restrict__ q, const T *__restrict__ k,
                      const T *__restrict__ v, const T *__restrict__ dout,
                      const float4 *__restrict__ rec, const uint32_t *__restrict__ off,
                      const int32_t *__restrict__ ent_row, const uint8_t *__restrict__ ent_slot,
                      float *__restrict__ dk, float *__restrict__ dv, float *__restrict__ dlmk) {
  constexpr int KPT = ChunkCfg<D>::kKeys, NT = ChunkCfg<D>::kThreads;
  constexpr int KS = kC / KPT;  // distance between a thread's keys
  constexpr int DQ = D / 4;     // dimensions per thread
  constexpr int DS = DQ + 4;    // stride of a staged quarter row: 16-byte aligned, and the
                                // four quarters a warp reads fall in distinct bank groups
  // the staged rows [row][quarter][DS] of q and dO
  __shared__ __align__(16) float qs[kRowBatch * 4 * DS], os[kRowBatch * 4 * DS];
  __shared__ float4 st[kRowBatch];
  __shared__ int own_s[kRowBatch];  // 1: the row's own chunk (slot k), with its position offset
  __shared__ int jmax_s[kRowBatch];
  const int seg = blockIdx.x;  // (b * Hkv + hkv) * nch + c
  const int c = seg % bs.nch, bk = seg / bs.nch;
  const int b = bk / bs.Hkv, hkv = bk % bs.Hkv;
  const int G = bs.Hq / bs.Hkv;
  const int L = bs.L, K = bs.topk;
  const int nkeys = min(kC, L - c * kC);
  const size_t krow0 = (size_t)bk * L + (size_t)c * kC;
  const int tid = threadIdx.x;
  const int jp = tid >> 2, qd = tid & 3;  // keys jp + kk * KS, dimension quarter qd
  // the thread's quarter of its keys' K and V rows, kept in registers (keys
  // past the chunk's end read its last key; their p is zero)
  float kr[KPT][DQ], vr[KPT][DQ];
#pragma unroll
  for (int kk = 0; kk < KPT; ++kk) {
    const size_t kj = (krow0 + min(jp + kk * KS, nkeys - 1)) * D + qd * DQ;
    ld_vec<T, DQ>(k + kj, kr[kk]);
    ld_vec<T, DQ>(v + kj, vr[kk]);
  }
  float ak[KPT][DQ], av[KPT][DQ];
#pragma unroll
  for (int kk = 0; kk < KPT; ++kk)
#pragma unroll
    for (int u = 0; u < DQ; ++u) ak[kk][u] = av[kk][u] = 0.0f;
  float al = 0.0f;  // dlmk: thread tid < D owns dimension tid
  // rows: own rows (every query head of the group, positions of this chunk),
  // then the rows that selected the chunk
  const int n_own = G * nkeys;
  const uint32_t s0 = off[seg], s1 = off[seg + 1];
  const int n_rows = n_own + (int)(s1 - s0);
  for (int r0 = 0; r0 < n_rows; r0 += kRowBatch) {
    const int nb = min(kRowBatch, n_rows - r0);
    __syncthreads();
    // stage the batch: 8 elements of a row per thread and step
    for (int i = tid; i < nb * (D / 8); i += NT) {
      const int rr = i / (D / 8), e = (i % (D / 8)) * 8;
      const int ri = r0 + rr;
      long long row;
      if (ri < n_own) {
        const int g = ri / nkeys, tt = ri % nkeys;
        row = ((long long)b * bs.Hq + hkv * G + g) * L + (long long)c * kC + tt;
      } else {
        row = ent_row[s0 + (ri - n_own)];
      }
      float f[8];
      const int at = (rr * 4 + e / DQ) * DS + e % DQ;
      ld8<T>(q + (size_t)row * D + e, f);
      *reinterpret_cast<float4 *>(qs + at) = make_float4(f[0], f[1], f[2], f[3]);
      *reinterpret_cast<float4 *>(qs + at + 4) = make_float4(f[4], f[5], f[6], f[7]);
      ld8<T>(dout + (size_t)row * D + e, f);
      *reinterpret_cast<float4 *>(os + at) = make_float4(f[0], f[1], f[2], f[3]);
      *reinterpret_cast<float4 *>(os + at + 4) = make_float4(f[4], f[5], f[6], f[7]);
      if (e == 0) {
        const int slot = ri < n_own ? K : (int)ent_slot[s0 + (ri - n_own)];
        st[rr] = rec[(size_t)row * (K + 1) + slot];
        own_s[rr] = ri < n_own ? 1 : 0;
        jmax_s[rr] = ri < n_own ? (ri % nkeys) : kC - 1;
      }
    }
    __syncthreads();
    for (int rr = 0; rr < nb; ++rr) {
      const float4 *qr = reinterpret_cast<const float4 *>(qs + (rr * 4 + qd) * DS);
      const float4 *orow = reinterpret_cast<const float4 *>(os + (rr * 4 + qd) * DS);
      float2 a2[KPT], d22[KPT];
#pragma unroll
      for (int kk = 0; kk < KPT; ++kk) a2[kk] = d22[kk] = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int u = 0; u < DQ / 4; ++u) {
        const float4 q4 = qr[u], o4 = orow[u];
#pragma unroll
        for (int kk = 0; kk < KPT; ++kk) {
          a2[kk] = __ffma2_rn(make_float2(q4.x, q4.y), make_float2(kr[kk][4 * u], kr[kk][4 * u + 1]), a2[kk]);
          a2[kk] = __ffma2_rn(make_float2(q4.z, q4.w), make_float2(kr[kk][4 * u + 2], kr[kk][4 * u + 3]), a2[kk]);
          d22[kk] = __ffma2_rn(make_float2(o4.x, o4.y), make_float2(vr[kk][4 * u], vr[kk][4 * u + 1]), d22[kk]);
          d22[kk] = __ffma2_rn(make_float2(o4.z, o4.w), make_float2(vr[kk][4 * u + 2], vr[kk][4 * u + 3]), d22[kk]);
        }
      }
      const float4 s4 = st[rr];  // lse_c, w_c, g_c, ds_c
      const bool own_r = own_s[rr] != 0;
      const int jm = jmax_s[rr];
      float2 dx2[KPT], pw2[KPT];
#pragma unroll
      for (int kk = 0; kk < KPT; ++kk) {
        float a = a2[kk].x + a2[kk].y, d2 = d22[kk].x + d22[kk].y;
        a += __shfl_xor_sync(0xffffffffu, a, 1);
        a += __shfl_xor_sync(0xffffffffu, a, 2);
        d2 += __shfl_xor_sync(0xffffffffu, d2, 1);
        d2 += __shfl_xor_sync(0xffffffffu, d2, 2);
        const int j = jp + kk * KS;
        const bool in = j < nkeys && j <= jm;
        const float pj = in ? __expf(a * bs.scale - s4.x) : 0.0f;
        const float dx = s4.y * pj * (d2 - s4.z) + (own_r ? pj * s4.w : 0.0f);
        const float pw = s4.y * pj;
        dx2[kk] = make_float2(dx, dx);
        pw2[kk] = make_float2(pw, pw);
      }
#pragma unroll
      for (int u = 0; u < DQ / 4; ++u) {
        const float4 q4 = qr[u], o4 = orow[u];
#pragma unroll
        for (int kk = 0; kk < KPT; ++kk) {
          float2 t;
          t = __ffma2_rn(pw2[kk], make_float2(o4.x, o4.y), make_float2(av[kk][4 * u], av[kk][4 * u + 1]));
          av[kk][4 * u] = t.x; av[kk][4 * u + 1] = t.y;
          t = __ffma2_rn(pw2[kk], make_float2(o4.z, o4.w), make_float2(av[kk][4 * u + 2], av[kk][4 * u + 3]));
          av[kk][4 * u + 2] = t.x; av[kk][4 * u + 3] = t.y;
          t = __ffma2_rn(dx2[kk], make_float2(q4.x, q4.y), make_float2(ak[kk][4 * u], ak[kk][4 * u + 1]));
          ak[kk][4 * u] = t.x; ak[kk][4 * u + 1] = t.y;
          t = __ffma2_rn(dx2[kk], make_float2(q4.z, q4.w), make_float2(ak[kk][4 * u + 2], ak[kk][4 * u + 3]));
          ak[kk][4 * u + 2] = t.x; ak[kk][4 * u + 3] = t.y;
        }
      }
      if (!own_r && tid < D) al = fmaf(s4.w, qs[(rr * 4 + tid / DQ) * DS + tid % DQ], al);
    }
  }
#pragma unroll
  for (int kk = 0; kk < KPT; ++kk) {
    const int j = jp + kk * KS;
    if (j < nkeys) {
      float *dkr = dk + (krow0 + j) * D + qd * DQ, *dvr = dv + (krow0 + j) * D + qd * DQ;
#pragma unroll
      for (int u = 0; u < DQ; u += 4) {
        *reinterpret_cast<float4 *>(dkr + u) =
            make_float4(ak[kk][u] * bs.scale, ak[kk][u + 1] * bs.scale, ak[kk][u + 2] * bs.scale,
                        ak[kk][u + 3] * bs.scale);
        *reinterpret_cast<float4 *>(dvr + u) =
            make_float4(av[kk][u], av[kk][u + 1], av[kk][u + 2], av[kk][u + 3]);
      }
    }
  }
  if (c < bs.nlmk && tid < D) dlmk[((size_t)bk * bs.nlmk + c) * D + tid] = al * bs.scale;
}

size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

BwdSpec bwd_spec(int B, int Hq, int Hkv, int L, int d, int topk, float scale) {
  BwdSpec bs{};
  bs.B = B;
  bs.Hq = Hq;
  bs.Hkv = Hkv;
  bs.L = L;
  bs.d = d;
  bs.topk = topk;
  bs.scale = scale;
  bs.nch = (L + kC - 1) / kC;
  bs.nlmk = L / kC;
  return bs;
}

size_t bwd_workspace_bytes(const BwdSpec &bs) {
  const size_t rows = (size_t)bs.B * bs.Hq * bs.L;
  const size_t nseg = (size_t)bs.B * bs.Hkv * bs.nch;
  size_t n = 256;                                    // error word
  n += al256(rows * (bs.topk + 1) * sizeof(float4)); // per-(row, slot) records
  n += al256(nseg * sizeof(uint32_t));               // counts / fill cursors
  n += al256((nseg + 1) * sizeof(uint32_t));         // segment offsets
  n += al256(rows * bs.topk * sizeof(int32_t));      // entries: rows
  n += al256(rows * bs.topk);                        // entries: slots
  return n;
}

cudaError_t bwd_run(const BwdSpec &bs, bool bf16, const void *q, const void *k, const void *v,
                    const void *lmk, const int32_t *sel, const float *chunk_w, const float *lse,
                    const void *dout, const float *dlse, float *dq, float *dk, float *dv,
                    float *dlmk, void *ws, uint32_t *err, cudaStream_t st, int *launches) {
  const size_t rows = (size_t)bs.B * bs.Hq * bs.L;
  const size_t nseg = (size_t)bs.B * bs.Hkv * bs.nch;
  unsigned char *p = static_cast<unsigned char *>(ws) + 256;
  auto take = [&](size_t bytes) {
    unsigned char *r = p;
    p += al256(bytes);
    return r;
  };
  float4 *rec = reinterpret_cast<float4 *>(take(rows * (bs.topk + 1) * sizeof(float4)));
  uint32_t *cnt = reinterpret_cast<uint32_t *>(take(nseg * sizeof(uint32_t)));
  uint32_t *off = reinterpret_cast<uint32_t *>(take((nseg + 1) * sizeof(uint32_t)));
  int32_t *ent_row = reinterpret_cast<int32_t *>(take(rows * bs.topk * sizeof(int32_t)));
  uint8_t *ent_slot = reinterpret_cast<uint8_t *>(take(rows * bs.topk));
  cudaError_t e;
  // the row pass counts the (row, slot) pairs per chunk
  if ((e = cudaMemsetAsync(cnt, 0, nseg * sizeof(uint32_t), st)) != cudaSuccess) return e;
  const unsigned rgrid = (unsigned)((rows + kRowWarps - 1) / kRowWarps);
#define HILS_BWD_ROWS(T, DD)                                                                     \
  bwd_rows_kernel<T, DD><<<rgrid, kRowWarps * 32, 0, st>>>(                                     \
      bs, (const T *)q, (const T *)k, (const T *)v, (const T *)lmk, sel, chunk_w, lse,           \
      (const T *)dout, dlse, rec, dq, cnt, err)
  if (bf16) { if (bs.d == 64) HILS_BWD_ROWS(__nv_bfloat16, 64); else HILS_BWD_ROWS(__nv_bfloat16, 128); }
  else { if (bs.d == 64) HILS_BWD_ROWS(float, 64); else HILS_BWD_ROWS(float, 128); }
#undef HILS_BWD_ROWS
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const long long nsel = (long long)rows * bs.topk;
  const unsigned sgrid = (unsigned)((nsel + 255) / 256);
  bwd_scan_kernel<<<1, 1024, 0, st>>>(cnt, off, (int)nseg);
  bwd_fill_kernel<<<sgrid, 256, 0, st>>>(bs, sel, off, cnt, ent_row, ent_slot);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
#define HILS_BWD_CHUNKS(T, DD)                                                                   \
  do {                                                                                           \
    auto kern = bwd_chunks_kernel<T, DD>;                                                        \
    kern<<<(unsigned)nseg, ChunkCfg<DD>::kThreads, 0, st>>>(bs, (const T *)q, (const T *)k,      \
        (const T *)v, (const T *)dout, rec, off, ent_row, ent_slot, dk, dv, dlmk);               \
  } while (0)
  if (bf16) { if (bs.d == 64) HILS_BWD_CHUNKS(__nv_bfloat16, 64); else HILS_BWD_CHUNKS(__nv_bfloat16, 128); }
  else { if (bs.d == 64) HILS_BWD_CHUNKS(float, 64); else HILS_BWD_CHUNKS(float, 128); }
#undef HILS_BWD_CHUNKS
  *launches += 4;
  return cudaGetLastError();
}

}  // namespace hils
