// Decode step of HiLS attention (one new query per head, position t = N-1 of
// a KV cache of length N that already holds the new token): landmark scoring,
// inter-chunk normaliser and top-k (model card "HiLS-Attention", section
// "What HiLS-Attention is"; molayo1419.me, "Core idea" step 1), then
// attention inside the selected chunks and the own chunk fused by the chunk
// logits (molayo1419.me step 2; aiweekly.co mechanism paragraph).
//
// The step is bound by HBM bytes: every landmark key of every (b, kv-head)
// and the K/V of the chunks the G = Hq/Hkv query heads of a KV head attend.
// The landmark rows stream through once for all G heads, and each chunk's
// K/V is staged once (bulk asynchronous copies into shared memory) for every
// head that attends it, so the union of the heads' chunks crosses HBM once.
//
//   decode_gemv_tc grid (min(ceil(n_c/128), 8), B*Hkv), bf16 and G <= 16:
//                  per 128-landmark tile one tcgen05.mma (M = 128 landmarks,
//                  N = 16 padded heads) -> the logits of the G heads, into a
//                  workspace array (decode_gemv: the same on the CUDA cores,
//                  one thread per landmark, for fp32 or G > 16)
//   decode_topk    grid (B*Hq): the head's log-sum-exp and exact top-k ->
//                  sel_idx / chunk_w, ascending chunk ids, lse_lmk.  The k-th
//                  largest of the 32-logit block maxima bounds the k-th
//                  largest logit from below; the logits at or above it are
//                  ranked exactly by (logit, chunk) keys (radix select on the
//                  logit bits when there are too many of them)
//   decode_union   grid (B*Hkv): the KV head's chunk union with a per-entry
//                  head mask and per-head logits
//   decode_attn    grid (Q, B*Hkv), 128 threads: up to 16 union chunks per
//                  CTA, each chunk's K and V staged once for all G heads (a
//                  thread per key for the logits, a thread per column pair
//                  for P V); per head an online (max, sum, acc) partial over
//                  its chunks.  With a page table the chunk's
//                  [64][d] slab of KV head hkv is read from its page
//                  ([num_pages][Hkv][64][d] pools) instead of the dense cache
//   decode_combine grid (B*Hq): partials -> out, lse
#include <cuda_bf16.h>

#include <algorithm>
#include <utility>

#include "common.cuh"
#include "kernels.h"
#include "paged.h"
#include "sm100.cuh"

namespace hils {
namespace {

// Programmatic dependent launch.  A kernel launched with the programmatic
// stream-serialization attribute may start while the kernel before it in the
// stream is still running; grid_dep_wait() returns once that kernel has
// completed and its writes are visible (at once for an ordinary launch), so
// everything before it may only read inputs no kernel in flight writes.
// grid_dep_launch() lets the next such kernel start launching once every
// block of this grid has called it or exited.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

using namespace sm100;

constexpr int kGemvThreads = 128; // landmarks per scoring CTA
constexpr int kChunksPerCta = 16; // union chunks per attention CTA
constexpr int kMaxG = 8;         // query heads per KV head handled per CTA
constexpr int kTkThreads = 512;  // top-k CTA (one head)
constexpr int kTkWarps = kTkThreads / 32;
constexpr int kC = 64;

__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes,
                                         uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// 8 consecutive elements through the read-only path, widened to fp32
template <typename T>
__device__ __forceinline__ void ldg8(const T *p, float (&f)[8]);
template <>
__device__ __forceinline__ void ldg8<__nv_bfloat16>(const __nv_bfloat16 *p, float (&f)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
template <>
__device__ __forceinline__ void ldg8<float>(const float *p, float (&f)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4 *>(p));
  const float4 b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

// Bounded wait on a single-use barrier (phase 0); sets *abort on timeout.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort) {
  return mbar_wait(bar, parity, abort);
}

// ---------------------------------------------------------------------------
// Landmark logits of the G query heads of one KV head: one thread per
// landmark, its row streamed from HBM with 16-byte loads all in flight, the
// scaled queries broadcast from shared memory.
template <typename T, int D>
__global__ void __launch_bounds__(kGemvThreads) decode_gemv_kernel(DecodeSpec ds,
                                                                  const T *__restrict__ q,
                                                                  const T *__restrict__ lmk,
                                                                  float *__restrict__ scores) {
  __shared__ __align__(16) float qs[kMaxG * D];  // [G][D], scaled
  const int G = ds.Hq / ds.Hkv;
  const int bk = blockIdx.y;
  const int b = bk / ds.Hkv, hkv = bk % ds.Hkv;
  for (int i = threadIdx.x; i < G * D; i += kGemvThreads) {
    const int g = i / D, e = i % D;
    qs[i] = to_f(q[((size_t)b * ds.Hq + hkv * G + g) * D + e]) * ds.scale;
  }
  __syncthreads();
  const int c = blockIdx.x * kGemvThreads + threadIdx.x;
  if (c >= ds.n_c) return;
  const T *row = lmk + ((size_t)bk * ds.nlmk + c) * D;
  float a[kMaxG];
#pragma unroll
  for (int g = 0; g < kMaxG; ++g) a[g] = 0.0f;
  // the row in two halves (registers), each half's loads issued together
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    constexpr int H = D / 2;
    float f[H];
#pragma unroll
    for (int cc = 0; cc < H / 8; ++cc) {
      float g8[8];
      ldg8<T>(row + half * H + cc * 8, g8);
#pragma unroll
      for (int u = 0; u < 8; ++u) f[cc * 8 + u] = g8[u];
    }
#pragma unroll
    for (int g = 0; g < kMaxG; ++g) {
      if (g < G) {
#pragma unroll
        for (int e = 0; e < H; e += 4) {
          const float4 qv = *reinterpret_cast<const float4 *>(qs + g * D + half * H + e);
          a[g] = fmaf(f[e], qv.x, a[g]);
          a[g] = fmaf(f[e + 1], qv.y, a[g]);
          a[g] = fmaf(f[e + 2], qv.z, a[g]);
          a[g] = fmaf(f[e + 3], qv.w, a[g]);
        }
      }
    }
  }
#pragma unroll
  for (int g = 0; g < kMaxG; ++g)
    if (g < G) scores[((size_t)bk * G + g) * ds.n_c + c] = a[g];
}

// Landmark logits on the tensor cores (bf16): per 128-landmark tile one
// MMA  S = Lmk_tile [128 x d] . Qg^T [d x 16], the G query heads of the KV
// head zero-padded to 16 rows, scaled after the fp32 accumulation (the same
// arithmetic as the prefill scoring kernel).  Warp 0 streams the tiles with
// TMA through a 3-stage ring, warp 1 issues the MMAs into two TMEM
// accumulators, warps 2-5 (one thread per landmark) write the G logits.
constexpr int kTcRows = 128;
constexpr int kTcStages = 3;
constexpr int kTcN = 16;  // padded head count (UMMA N)
constexpr int kTcTilesPerCta = 8;

template <int D>
struct GemvTcLayout {
  static constexpr int kTileBytes = kTcRows * D * 2;
  static constexpr int ring = 0;
  static constexpr int bq = ring + kTcStages * kTileBytes;  // Q^T: [D/64][16 rows][128 B]
  static constexpr int bars = bq + (D / 64) * kTcN * 128;
  static constexpr int misc = bars + 16 * 8;
  static constexpr int total = misc + 16;
};

struct GemvTcBars {
  uint64_t full[kTcStages], empty[kTcStages], acc_full[2], acc_empty[2], done;
};

template <int D>
__global__ void __launch_bounds__(192, 1)
    decode_gemv_tc_kernel(const __grid_constant__ CUtensorMap tm_l, DecodeSpec ds,
                          const __nv_bfloat16 *__restrict__ q, float *__restrict__ scores,
                          uint32_t *__restrict__ err) {
  using Lay = GemvTcLayout<D>;
  grid_dep_launch();  // the top-k may launch (it waits for this grid's scores)
  // a name of its own: this kernel asks the dynamic window for 1024-byte alignment
  extern __shared__ __align__(1024) unsigned char smem_tc[];
  unsigned char *smem = smem_tc;
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) report(err, DEV_BAD_INDEX);
    return;
  }
  GemvTcBars *bars = reinterpret_cast<GemvTcBars *>(smem + Lay::bars);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Lay::misc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Lay::misc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = ds.Hq / ds.Hkv;
  const int bk = blockIdx.y, b = bk / ds.Hkv, hkv = bk % ds.Hkv;
  const int ntiles = (ds.n_c + kTcRows - 1) / kTcRows;
  const int my_n =
      ntiles > (int)blockIdx.x ? (ntiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->acc_full[i], 1);
      mbar_init(&bars->acc_empty[i], kTcRows);
    }
    mbar_init(&bars->done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) prefetch_tmap(&tm_l);
  if (warp == 1) {
    tmem_alloc(tmem_slot, 32);  // two 16-column accumulators
    tmem_relinquish();
  }
  // Q^T tile (K-major, 128-byte swizzle): row g = head g's query, 0 past G
  for (int i = threadIdx.x; i < kTcN * D; i += blockDim.x) {
    const int g = i / D, d = i % D;
    const __nv_bfloat16 val =
        g < G ? q[((size_t)b * ds.Hq + hkv * G + g) * D + d] : __float2bfloat16(0.0f);
    const int kb = d >> 6, c = d & 63;
    const int off = kb * kTcN * 128 + g * 128 + ((((c >> 3) ^ (g & 7))) << 4) + (c & 7) * 2;
    *reinterpret_cast<__nv_bfloat16 *>(smem + Lay::bq + off) = val;
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < my_n; ++i) {
        const int tile = blockIdx.x + i * gridDim.x, s = i % kTcStages;
        if (i >= kTcStages && !mbar_wait(&bars->empty[s], ((i / kTcStages) - 1) & 1, abort_flag))
          break;
        mbar_expect_tx(&bars->full[s], Lay::kTileBytes);
        unsigned char *dst = smem + Lay::ring + s * Lay::kTileBytes;
        for (int kb = 0; kb < D / 64; ++kb)
          tma_load_2d(dst + kb * kTcRows * 128, &tm_l, &bars->full[s], kb * 64,
                      bk * ds.nlmk + tile * kTcRows);
        ++issued;
      }
      for (int i = (issued > kTcStages ? issued - kTcStages : 0); i < issued; ++i)
        mbar_wait_bounded(&bars->full[i % kTcStages], (i / kTcStages) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kTcRows, kTcN, false, false);
      const uint32_t bq_addr = smem_u32(smem + Lay::bq);
      for (int i = 0; i < my_n; ++i) {
        const int s = i % kTcStages, ab = i & 1;
        if (!mbar_wait(&bars->full[s], (i / kTcStages) & 1, abort_flag)) break;
        if (i >= 2 && !mbar_wait(&bars->acc_empty[ab], ((i >> 1) - 1) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + Lay::ring + s * Lay::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int kb = kk >> 2, kw = kk & 3;
          const uint64_t ad = smem_desc_sw128(a_addr + kb * kTcRows * 128 + kw * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(bq_addr + kb * kTcN * 128 + kw * 32, 16, 1024);
          mma_bf16_ss(tmem + ab * kTcN, ad, bd, idesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars->acc_full[ab]);
        mma_commit(&bars->empty[s]);
      }
      mma_commit(&bars->done);
      mbar_wait_bounded(&bars->done, 0);
    }
  } else {
    const int r = 32 * (warp & 3) + lane;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    for (int i = 0; i < my_n; ++i) {
      const int ab = i & 1, tile = blockIdx.x + i * gridDim.x;
      const bool ok = mbar_wait(&bars->acc_full[ab], (i >> 1) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      float v[16];
      tmem_ld16(tmem + ab * kTcN + lane_off, v);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bars->acc_empty[ab]);
      const int c = tile * kTcRows + r;
      if (c < ds.n_c) {
#pragma unroll
        for (int g = 0; g < kTcN; ++g)
          if (g < G) scores[((size_t)bk * G + g) * ds.n_c + c] = v[g] * ds.scale;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) report(err, DEV_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 32);
  }
}

// order-preserving 32-bit image of an fp32 score (-0 folded into +0)
__device__ __forceinline__ uint32_t score_bits(float s) {
  uint32_t x = __float_as_uint(s + 0.0f);
  return (x & 0x80000000u) ? ~x : (x | 0x80000000u);
}

// Exact top-k of one head's landmark logits (s desc, c asc) and their
// log-sum-exp.  The k-th largest score is found by a radix select on the
// order-preserving bits (four 8-bit digits, per-warp histograms); the kept
// chunks are then written in ascending chunk order, the lowest ids among
// scores equal to the k-th.
__global__ void __launch_bounds__(kTkThreads) decode_topk_kernel(DecodeSpec ds,
                                                          const float *__restrict__ scores,
                                                          int32_t *__restrict__ sel,
                                                          float *__restrict__ chunk_w,
                                                          float *__restrict__ lse_lmk,
                                                          int staged) {
  extern __shared__ __align__(16) float sc_s[];  // the head's logits when staged
  // digit histograms (one per pair of warps); also read as 64-bit candidate
  // keys, hence the alignment
  __shared__ __align__(16) uint32_t hist_w[8 * 256];
  __shared__ uint32_t hist[256];
  __shared__ int wsum[kTkWarps];
  __shared__ float red[kTkWarps];
  __shared__ uint32_t s_prefix, s_bin;
  __shared__ int s_need;
  const int h = blockIdx.x;  // b*Hq + hq
  const int n = ds.n_c, K = ds.topk;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float *sc = scores + (size_t)h * n;
  grid_dep_launch();
  grid_dep_wait();  // the landmark pass's scores
  if (staged) {
    // one pass over HBM/L2 with every load in flight; the rest reads shared memory
#pragma unroll 8
    for (int i = tid; i < n; i += kTkThreads) sc_s[i] = sc[i];
    __syncthreads();
    sc = sc_s;
  }
  int32_t *srow = sel + (size_t)h * K;
  float *wrow = chunk_w + (size_t)h * K;

  // log-sum-exp: block maximum, then the sum of exponentials against it
  float m = -INFINITY;
#pragma unroll 8
  for (int i = tid; i < n; i += kTkThreads) m = fmaxf(m, sc[i]);
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  m = red[0];
#pragma unroll
  for (int w = 1; w < kTkWarps; ++w) m = fmaxf(m, red[w]);
  __syncthreads();
  float l = 0.0f;
  if (n > 0) {
#pragma unroll 8
    for (int i = tid; i < n; i += kTkThreads) l += __expf(sc[i] - m);
  }
  for (int o = 16; o; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  if (lane == 0) red[warp] = l;
  __syncthreads();
  if (tid == 0 && lse_lmk) {
    float lt = 0.0f;
    for (int w = 0; w < kTkWarps; ++w) lt += red[w];
    lse_lmk[h] = n > 0 ? m + __logf(lt) : -INFINITY;
  }

  if (n <= K) {
    // every completed chunk is selected
    for (int i = tid; i < K; i += kTkThreads) {
      srow[i] = i < n ? i : -1;
      wrow[i] = i < n ? sc[i] : -INFINITY;
    }
    return;
  }
  // Threshold path (staged logits, at least k blocks of 32): the k-th largest
  // block maximum tau bounds the k-th largest logit from below (the k best
  // blocks hold k distinct logits >= tau), so every kept chunk is among the
  // few logits >= tau; their exact top-k by (logit desc, chunk asc) is taken
  // by counting, then written in chunk order through a bitmap.
  const int nb = (n + 31) / 32;
  constexpr int kCandCap = 8 * 256 / 2;  // 64-bit candidate keys in hist_w
  if (staged && nb >= K && nb <= 256) {
    uint32_t *bmax = hist;  // [256] block maxima (order-preserving bits)
    uint64_t *cand = reinterpret_cast<uint64_t *>(hist_w);
    __shared__ int n_cand_s;
    __shared__ uint32_t tau_s;
    __shared__ uint32_t keep[256];  // one bit per chunk (n <= 8192)
    if (tid == 0) n_cand_s = 0;
    if (tid < 256) keep[tid] = 0u;
    // block maxima: two threads per block, 16 logits each in a lane-rotated
    // order (no bank conflicts), combined across the pair
    // (whole warps take part, for the pair shuffles; act: the pair's block exists)
    const int pair_warps_end = (2 * nb + 31) & ~31;
    if (tid < pair_warps_end) {
      const int bk = tid >> 1, hf = tid & 1;
      const bool act = bk < nb;
      uint32_t m = 0u;
#pragma unroll 8
      for (int u = 0; u < 16; ++u) {
        const int i = bk * 32 + hf * 16 + ((u + bk) & 15);
        if (act && i < n) m = max(m, score_bits(sc[i]));
      }
      m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
      if (act && hf == 0) bmax[bk] = m;
    }
    __syncthreads();
    if (tid < pair_warps_end) {
      // rank of this block's maximum (ties: lower block first), the pair
      // splitting the other blocks between them
      const int bk = tid >> 1, hf = tid & 1;
      const bool act = bk < nb;
      const uint32_t v = act ? bmax[bk] : 0u;
      int rank = 0;
      if (act) {
#pragma unroll 8
        for (int b2 = hf; b2 < nb; b2 += 2) {
          const uint32_t x = bmax[b2];
          rank += (x > v || (x == v && b2 < bk)) ? 1 : 0;
        }
      }
      rank += __shfl_xor_sync(0xffffffffu, rank, 1);
      if (act && hf == 0 && rank == K - 1) tau_s = v;
    }
    __syncthreads();
    const uint32_t tau = tau_s;
    // candidates: only a block whose maximum reaches tau holds any; a warp
    // per such block, one lane per logit
    for (int b2 = warp; b2 < nb; b2 += kTkWarps) {
      if (bmax[b2] < tau) continue;
      const int i = b2 * 32 + lane;
      const uint32_t kb = i < n ? score_bits(sc[i]) : 0u;
      const bool in = i < n && kb >= tau;
      const uint32_t bal = __ballot_sync(0xffffffffu, in);
      int base = 0;
      if (lane == 0) base = atomicAdd(&n_cand_s, __popc(bal));
      base = __shfl_sync(0xffffffffu, base, 0);
      const int pos = base + __popc(bal & ((1u << lane) - 1u));
      if (in && pos < kCandCap) cand[pos] = ((uint64_t)kb << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)i);
    }
    __syncthreads();
    const int m = n_cand_s;
    if (m <= kCandCap) {
      // exact rank of every candidate key; the k best are kept
      for (int a = tid; a < m; a += kTkThreads) {
        const uint64_t x = cand[a];
        int rank = 0;
#pragma unroll 8
        for (int b2 = 0; b2 < m; ++b2) rank += cand[b2] > x ? 1 : 0;
        if (rank < K) {
          const int i = (int)(0xFFFFFFFFu - (uint32_t)x);
          atomicOr(&keep[i >> 5], 1u << (i & 31));
        }
      }
      __syncthreads();
      // write in chunk order: word w's kept chunks go after those of words < w
      if (warp == 0) {
        int carry = 0;
        for (int w0 = 0; w0 < 256; w0 += 32) {
          const uint32_t word = keep[w0 + lane];
          const int c1 = __popc(word);
          int x = c1;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
          }
          int pos = carry + x - c1;
          uint32_t wd = word;
          while (wd) {
            const int i = (w0 + lane) * 32 + __ffs(wd) - 1;
            wd &= wd - 1;
            if (pos < K) {
              srow[pos] = i;
              wrow[pos] = sc[i];
            }
            ++pos;
          }
          carry += __shfl_sync(0xffffffffu, x, 31);
        }
      }
      return;
    }
    // too many candidates (logits crowding at tau): the radix select below
    __syncthreads();
  }
  // radix select of the K-th largest key: per pass a histogram of one 8-bit
  // digit of the keys that match the digits chosen so far (one histogram per
  // warp, summed), then warp 0 finds the digit holding the need-th largest
  uint32_t prefix = 0;
  int need = K;
  uint32_t last_bin = 0;  // keys equal to the final prefix
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < 8 * 256; i += kTkThreads) hist_w[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += kTkThreads) {
      const uint32_t k = score_bits(sc[i]);
      if (pass == 0 || (k >> (shift + 8)) == prefix) atomicAdd(&hist_w[(warp & 7) * 256 + ((k >> shift) & 255u)], 1u);
    }
    __syncthreads();
    if (tid < 256) {
      uint32_t sum = 0;
#pragma unroll
      for (int w = 0; w < 8; ++w) sum += hist_w[w * 256 + tid];
      hist[tid] = sum;
    }
    __syncthreads();
    if (warp == 0) {
      // bins from the top: lane j holds bins 255-8j .. 248-8j
      uint32_t cnt[8], tot = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        cnt[u] = hist[255 - 8 * lane - u];
        tot += cnt[u];
      }
      uint32_t incl = tot;
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t excl = incl - tot;
      // the lane whose range holds the need-th largest key
      if (excl < (uint32_t)need && incl >= (uint32_t)need) {
        uint32_t cum = excl;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (cum + cnt[u] >= (uint32_t)need && cum < (uint32_t)need) {
            s_prefix = (prefix << 8) | (uint32_t)(255 - 8 * lane - u);
            s_need = need - (int)cum;
            s_bin = cnt[u];
          }
          cum += cnt[u];
        }
      }
    }
    __syncthreads();
    prefix = s_prefix;
    need = s_need;
    last_bin = s_bin;
    __syncthreads();
  }
  // prefix = the K-th largest key T.  Kept: every key above T and the `need`
  // lowest chunk ids among the last_bin keys equal to T, written in ascending
  // chunk order.  Each warp owns a contiguous segment of the chunks; counts
  // per segment give every warp its output offset, then it writes in order.
  const uint32_t T = prefix;
  const bool all_eq = last_bin == (uint32_t)need;
  const int seg = (n + kTkWarps - 1) / kTkWarps;
  const int lo = warp * seg, hi = min(n, lo + seg);
  auto key_at = [&](int i) { return score_bits(sc[i]); };
  int my_eq = 0;
  if (!all_eq)
    for (int i0 = lo; i0 < hi; i0 += 32) {
      const int i = i0 + lane;
      my_eq += __popc(__ballot_sync(0xffffffffu, i < hi && key_at(i) == T));
    }
  if (lane == 0) wsum[warp] = my_eq;
  __syncthreads();
  int eq_before = 0;
#pragma unroll
  for (int w = 0; w < kTkWarps; ++w) eq_before += w < warp ? wsum[w] : 0;
  __syncthreads();
  // takes per segment
  int my_take = 0;
  {
    int eq_run = eq_before;
    for (int i0 = lo; i0 < hi; i0 += 32) {
      const int i = i0 + lane;
      const uint32_t k = i < hi ? key_at(i) : 0u;
      const bool gt = i < hi && k > T, eq = i < hi && k == T;
      const uint32_t eqb = __ballot_sync(0xffffffffu, eq);
      const int rank = eq_run + __popc(eqb & ((1u << lane) - 1u));
      const bool take = gt || (eq && (all_eq || rank < need));
      my_take += __popc(__ballot_sync(0xffffffffu, take));
      eq_run += __popc(eqb);
    }
  }
  if (lane == 0) wsum[warp] = my_take;
  __syncthreads();
  int base = 0;
#pragma unroll
  for (int w = 0; w < kTkWarps; ++w) base += w < warp ? wsum[w] : 0;
  {
    int eq_run = eq_before;
    for (int i0 = lo; i0 < hi; i0 += 32) {
      const int i = i0 + lane;
      const float v = i < hi ? sc[i] : 0.0f;
      const uint32_t k = i < hi ? score_bits(v) : 0u;
      const bool gt = i < hi && k > T, eq = i < hi && k == T;
      const uint32_t eqb = __ballot_sync(0xffffffffu, eq);
      const int rank = eq_run + __popc(eqb & ((1u << lane) - 1u));
      const bool take = gt || (eq && (all_eq || rank < need));
      const uint32_t tb = __ballot_sync(0xffffffffu, take);
      const int pos = base + __popc(tb & ((1u << lane) - 1u));
      if (take && pos < K) {
        srow[pos] = i;
        wrow[pos] = v;
      }
      base += __popc(tb);
      eq_run += __popc(eqb);
    }
  }
}

// ---------------------------------------------------------------------------
// The KV head's chunk union: the selections of its G query heads and the own
// chunk, ascending, with a per-entry mask of the heads that attend it and
// their logits.
__global__ void __launch_bounds__(256) decode_union_kernel(DecodeSpec ds,
                                                           const int32_t *__restrict__ sel,
                                                           const float *__restrict__ chunk_w,
                                                           int32_t *__restrict__ u_c,
                                                           uint32_t *__restrict__ u_mask,
                                                           float *__restrict__ u_logit,
                                                           int32_t *__restrict__ u_count) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int G = ds.Hq / ds.Hkv, K = ds.topk;
  uint64_t *chosen = reinterpret_cast<uint64_t *>(smem);          // [G][K]
  uint32_t *bitmap = reinterpret_cast<uint32_t *>(chosen + G * K);  // [nwords]
  int *prefix = reinterpret_cast<int *>(bitmap + ds.nwords);       // [nwords]
  __shared__ int total;
  const int bk = blockIdx.x;
  const int b = bk / ds.Hkv, hkv = bk % ds.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int own = ds.own;

  for (int i = tid; i < ds.nwords; i += blockDim.x) bitmap[i] = 0;
  grid_dep_launch();
  grid_dep_wait();  // the top-k's selections
  __syncthreads();
  for (int i = tid; i < G * K; i += blockDim.x) {
    const int g = i / K, j = i % K;
    const size_t hrow = (size_t)b * ds.Hq + hkv * G + g;
    const int c = sel[hrow * K + j];
    const bool have = c >= 0 && c < ds.n_c;
    chosen[i] = have ? sel_key(chunk_w[hrow * K + j], c) : 0ull;
    if (have) atomicOr(&bitmap[c >> 5], 1u << (c & 31));
  }
  __syncthreads();
  if (tid == 0) atomicOr(&bitmap[own >> 5], 1u << (own & 31));
  __syncthreads();
  // union positions: exclusive prefix of the bitmap popcounts (one warp)
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < ds.nwords; base += 32) {
      const int i = base + lane;
      const int c = i < ds.nwords ? __popc(bitmap[i]) : 0;
      int x = c;
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (i < ds.nwords) prefix[i] = carry + x - c;
      carry += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) total = carry;
  }
  __syncthreads();
  const int cap = ds.ucap;
  int32_t *uc = u_c + (size_t)bk * cap;
  uint32_t *um = u_mask + (size_t)bk * cap;
  float *ul = u_logit + (size_t)bk * cap * G;
  for (int i = tid; i < total; i += blockDim.x) um[i] = 0;
  __syncthreads();
  auto pos_of = [&](int c) {
    return prefix[c >> 5] + __popc(bitmap[c >> 5] & ((1u << (c & 31)) - 1u));
  };
  for (int i = tid; i < G * K; i += blockDim.x) {
    const int g = i / K;
    const uint64_t x = chosen[i];
    if (!x) continue;
    const int c = key_chunk(x);
    const int pos = pos_of(c);
    uc[pos] = c;
    atomicOr(&um[pos], 1u << g);
    ul[pos * G + g] = key_score(x);
  }
  __syncthreads();
  if (tid == 0) {
    const int pos = pos_of(own);
    uc[pos] = own;
    um[pos] = (1u << G) - 1u;  // every head attends its own chunk
    u_count[bk] = total;
  }
}

// ---------------------------------------------------------------------------
// Chunk attention of the union.  CTA (qi, bk) takes union entries
// [16 qi, 16 qi + 16) of (b, kv-head) bk; each chunk's K and V are copied
// into shared memory once (double-buffered bulk copies: the next chunk in
// flight while this one is used) and serve all G query heads of the KV head.
//   logits   thread t: key j = t mod 64 and part t / 64 of the head
//            dimension; K arrives as 128-byte-swizzled tiles of a 2-D tensor
//            copy, so the 8 lanes of a shared-memory wavefront, reading the
//            same 16-byte column chunk of 8 consecutive rows, find it at 8
//            different bank groups; the scaled queries are broadcast, all
//            heads accumulate in fp32 pairs, and the parts meet in shared
//            memory
//   softmax  warp w takes heads w, w + 4: the chunk's maximum and sum per
//            head, the probabilities stored key-major [64][GB]
//   P V      thread t: columns (2p, 2p+1), p = t mod (D/2), over key slice
//            t / (D/2), every head at once (pairs of heads per fp32x2 FMA)
// A running (max, sum, acc) per head merges the chunks under their fusion
// logits; the key slices are summed at the end into one partial record
// [M, L, acc[D]] per (bk, qi, g).
#ifndef HILS_DECODE_THREADS
#define HILS_DECODE_THREADS 256
#endif
constexpr int kAttnThreads = HILS_DECODE_THREADS;
#ifndef HILS_DECODE_MINB
#define HILS_DECODE_MINB 3
#endif
constexpr int kDimParts = kAttnThreads / 64;  // a key's dot product split over this many threads
#ifndef HILS_DECODE_STAGES
#define HILS_DECODE_STAGES 2
#endif
constexpr int kStages = HILS_DECODE_STAGES;  // chunk buffers per CTA (kStages - 1 copies ahead)

template <typename T, int D, int GB>
struct DecAttnLayout {
  static constexpr int kRow = D * (int)sizeof(T);        // bytes of one K or V row
  static constexpr int kBoxes = kRow / 128;              // 128-byte column boxes of K
  static constexpr int kKBuf = kC * kRow;                // one chunk's K tiles [kBoxes][64][128]
  // buffers: kStages, or as many as fit (fp32 rows are twice as long)
  static constexpr int kFit = (227 * 1024 - 16 * 1024) / (2 * kKBuf);
  static constexpr int kNS = kStages < kFit ? kStages : (kFit < 2 ? 2 : kFit);
  static constexpr int ks = 0;                           // K tiles [kNS][kKBuf]
  static constexpr int vs = ks + kNS * kKBuf;            // V slabs [kNS][64][kRow]
  static constexpr int qs = vs + kNS * kC * kRow;        // queries [GB][D] fp32, scaled
  static constexpr int xs = qs + GB * D * 4;             // partial logits [kDimParts][GB][64]
  static constexpr int ps = xs + kDimParts * GB * kC * 4;  // probabilities [64][GB]
  static constexpr int st = ps + kC * GB * 4;            // per head m, l, fusion logit, -
  static constexpr int bars = st + GB * 16;              // kNS mbarriers
  static constexpr int misc = bars + kNS * 8;            // abort flag
  // the CTA's union entries, read once: chunk, head mask, first K row (-1:
  // page outside the pool), element offset of the K / V slab, logits [GB]
  static constexpr int ent_c = misc + 16;
  static constexpr int ent_m = ent_c + kChunksPerCta * 4;
  static constexpr int ent_y = ent_m + kChunksPerCta * 4;
  static constexpr int ent_off = ent_y + kChunksPerCta * 4;
  static constexpr int ent_l = ent_off + kChunksPerCta * 8;
  static constexpr int total = ent_l + kChunksPerCta * GB * 4;
  static_assert(kKBuf % 1024 == 0, "swizzled tiles are 1024-byte aligned");
  static_assert(total <= 227 * 1024, "shared memory");
  // the key-slice sums at the end reuse the K tiles
  static_assert((kAttnThreads / (D / 2)) * GB * D * 4 <= kNS * kKBuf, "reduction area");
};

template <typename T, int D, int GB>
__global__ void __launch_bounds__(kAttnThreads, HILS_DECODE_MINB) decode_attn_kernel(
    const __grid_constant__ CUtensorMap tm_k, DecodeSpec ds, const T *__restrict__ q,
    const T *__restrict__ kc, const T *__restrict__ vc, const PagedKV pg, const int32_t *__restrict__ u_c,
    const uint32_t *__restrict__ u_mask, const float *__restrict__ u_logit,
    const int32_t *__restrict__ u_count, float *__restrict__ part, uint32_t *__restrict__ err) {
  using Lay = DecAttnLayout<T, D, GB>;
  constexpr int NS = Lay::kNS;  // chunk buffers: NS - 1 copies in flight ahead
  // a name of its own: this kernel asks the dynamic window for 1024-byte alignment
  extern __shared__ __align__(1024) unsigned char smem_at[];
  unsigned char *smem = smem_at;
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) report(err, DEV_BAD_INDEX);
    grid_dep_wait();  // complete only after the kernels before it (the next ones rely on that)
    return;
  }
  float *qs = reinterpret_cast<float *>(smem + Lay::qs);
  float *xs = reinterpret_cast<float *>(smem + Lay::xs);
  float *ps = reinterpret_cast<float *>(smem + Lay::ps);
  float *st = reinterpret_cast<float *>(smem + Lay::st);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Lay::bars);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Lay::misc);

  const int G = ds.Hq / ds.Hkv;
  const int qi = blockIdx.x, bk = blockIdx.y;
  const int b = bk / ds.Hkv, hkv = bk % ds.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cap = ds.ucap;
  const size_t kvbase = (size_t)bk * ds.N;
  const int t = ds.N - 1, own = ds.own;

  if (tid == 0) {
    *abort_flag = 0;
    for (int st2 = 0; st2 < NS; ++st2) mbar_init(&bars[st2], 1);
    fence_mbar_init();
    prefetch_tmap(&tm_k);
  }
  for (int i = tid; i < GB * D; i += kAttnThreads) {
    const int g = i / D, e = i % D;
    qs[i] = g < G ? to_f(q[((size_t)b * ds.Hq + hkv * G + g) * D + e]) * ds.scale : 0.0f;
  }
  for (int i = tid; i < kC * GB; i += kAttnThreads) ps[i] = 0.0f;  // heads >= G stay 0
  grid_dep_launch();
  grid_dep_wait();  // the union (everything above reads inputs only)
  const int count = u_count[bk];
  const int i0 = qi * kChunksPerCta, i1 = min(count, i0 + kChunksPerCta);
  int *ent_c = reinterpret_cast<int *>(smem + Lay::ent_c);
  uint32_t *ent_m = reinterpret_cast<uint32_t *>(smem + Lay::ent_m);
  int *ent_y = reinterpret_cast<int *>(smem + Lay::ent_y);
  size_t *ent_off = reinterpret_cast<size_t *>(smem + Lay::ent_off);
  float *ent_l = reinterpret_cast<float *>(smem + Lay::ent_l);
  if (tid < i1 - i0) {
    const size_t ue = (size_t)bk * cap + i0 + tid;
    const int c = u_c[ue];
    size_t off = (kvbase + (size_t)c * kC) * D;  // element offset of the chunk's [rows][D] slab
    int y = (int)(kvbase + (size_t)c * kC);       // its first row in the K tensor map
    if (pg.table) {
      // paged: the chunk is page table[b][c], its KV head hkv at [page][hkv][C][D]
      const long long page = pg.table[(size_t)b * pg.max_pages + c];
      const bool in_pool = page >= 0 && page < pg.num_pages;
      off = in_pool ? ((size_t)page * ds.Hkv + hkv) * kC * D : 0;
      y = in_pool ? (int)(((size_t)page * ds.Hkv + hkv) * kC) : -1;
    }
    ent_c[tid] = c;
    ent_m[tid] = u_mask[ue];
    ent_y[tid] = y;
    ent_off[tid] = off;
    for (int g = 0; g < G; ++g) ent_l[tid * GB + g] = u_logit[ue * G + g];
  }
  __syncthreads();
  // the copies of union entry i into buffer buf (thread 0): K as kBoxes
  // swizzled [64 rows][128 bytes] tiles (a partial last chunk reads rows
  // past the cache's end, never used), V as one slab of its valid rows
  auto issue = [&](int i, int buf) {
    const int li = i - i0;
    const int rows = min(kC, ds.N - ent_c[li] * kC);
    const int y = ent_y[li];
    if (y < 0) {
      // no copy for a page outside the pool: complete the phase without
      // bytes (the chunk's logits are then unspecified) and report it
      report(err, DEV_BAD_INDEX);
      mbar_expect_tx(&bars[buf], 0);
      return;
    }
    const size_t off = ent_off[li];
    mbar_expect_tx(&bars[buf], (uint32_t)(kC + rows) * Lay::kRow);
    unsigned char *kd = smem + Lay::ks + buf * Lay::kKBuf;
#pragma unroll
    for (int bx = 0; bx < Lay::kBoxes; ++bx)
      tma_load_2d(kd + bx * kC * 128, &tm_k, &bars[buf], bx * (128 / (int)sizeof(T)), y);
    bulk_g2s(smem + Lay::vs + buf * kC * Lay::kRow, vc + off, (uint32_t)rows * Lay::kRow,
             &bars[buf]);
  };
  // the first NS - 1 entries in flight before the loop
  if (tid == 0)
    for (int i = i0; i < min(i1, i0 + NS - 1); ++i) issue(i, (i - i0) % NS);

  constexpr int NP = D / 2;                  // column pairs
  constexpr int KS = kAttnThreads / NP;      // key slices of the P V pass
  constexpr int KPS = kC / KS;               // keys per slice
  constexpr int GP = GB >= 2 ? GB / 2 : 1;   // head pairs
  const int pcol = tid % NP, ksl = tid / NP;
  // acc for columns 2 pcol (a) and 2 pcol + 1 (b), heads (2 gp, 2 gp + 1) per pair
  float2 acc_a[GP], acc_b[GP];
#pragma unroll
  for (int gp = 0; gp < GP; ++gp) acc_a[gp] = acc_b[gp] = make_float2(0.0f, 0.0f);
  float Mr[GB], Lr[GB];
#pragma unroll
  for (int g = 0; g < GB; ++g) { Mr[g] = -INFINITY; Lr[g] = 0.0f; }

  bool ok = true;
  for (int i = i0; i < i1; ++i) {
    const int buf = (i - i0) % NS;
    // entry i + NS - 1 into the buffer entry i - 1 used (released by
    // the end-of-iteration barrier)
    if (tid == 0 && i + NS - 1 < i1) issue(i + NS - 1, (i + NS - 1 - i0) % NS);
    ok = __syncthreads_and(wait_bar(&bars[buf], ((i - i0) / NS) & 1, abort_flag));
    if (!ok) {
      // drain: every copy issued must land before the CTA exits
      if (tid == 0)
        for (int k2 = i; k2 < min(i1, i + NS); ++k2)
          mbar_wait_bounded(&bars[(k2 - i0) % NS], ((k2 - i0) / NS) & 1);
      break;
    }
    const int c = ent_c[i - i0];
    const uint32_t mask = ent_m[i - i0];
    const int jmax = (c == own) ? (t - c * kC) : (kC - 1);
    // ---- logits: partial dot products of key j with every head over part h of the dimension
    {
      const int j = tid & (kC - 1), h = tid >> 6;      // key, part of the head dimension
      constexpr int kDP = D / kDimParts;                 // dimensions per part
      const unsigned char *kr = smem + Lay::ks + buf * Lay::kKBuf + j * 128;
      const float *qh = qs + h * kDP;
      constexpr int kE = 16 / (int)sizeof(T);            // elements per 16-byte read
      constexpr int kSteps = kDP / kE;
      float2 a2[GB];
#pragma unroll
      for (int g = 0; g < GB; ++g) a2[g] = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int s2 = 0; s2 < kSteps; ++s2) {
        const int cabs = h * kSteps + s2;  // 16-byte chunk of the row: box cabs / 8, column cabs % 8
        const uint4 w = *reinterpret_cast<const uint4 *>(
            kr + (cabs >> 3) * (kC * 128) + (((cabs & 7) ^ (j & 7)) << 4));
        float f[kE];
        if constexpr (sizeof(T) == 2) {
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            f[2 * u] = __uint_as_float(ww[u] << 16);
            f[2 * u + 1] = __uint_as_float(ww[u] & 0xFFFF0000u);
          }
        } else {
          f[0] = __uint_as_float(w.x);
          f[1] = __uint_as_float(w.y);
          f[2] = __uint_as_float(w.z);
          f[3] = __uint_as_float(w.w);
        }
#pragma unroll
        for (int g = 0; g < GB; ++g) {
#pragma unroll
          for (int u4 = 0; u4 < kE / 4; ++u4) {
            const float4 qq = *reinterpret_cast<const float4 *>(qh + g * D + s2 * kE + 4 * u4);
            a2[g] = __ffma2_rn(make_float2(f[4 * u4], f[4 * u4 + 1]), make_float2(qq.x, qq.y), a2[g]);
            a2[g] = __ffma2_rn(make_float2(f[4 * u4 + 2], f[4 * u4 + 3]), make_float2(qq.z, qq.w), a2[g]);
          }
        }
      }
      float *xh = xs + h * GB * kC;
#pragma unroll
      for (int g = 0; g < GB; ++g) xh[g * kC + j] = a2[g].x + a2[g].y;
    }
    __syncthreads();
    // ---- per head: chunk maximum and sum, probabilities e_j = exp(x_j - m)
    for (int g = warp; g < G; g += kAttnThreads / 32) {
      if (!((mask >> g) & 1u)) {
        ps[lane * GB + g] = 0.0f;
        ps[(lane + 32) * GB + g] = 0.0f;
        continue;
      }
      float x0 = 0.0f, x1 = 0.0f;
#pragma unroll
      for (int h = 0; h < kDimParts; ++h) {
        x0 += xs[(h * GB + g) * kC + lane];
        x1 += xs[(h * GB + g) * kC + lane + 32];
      }
      x0 = lane <= jmax ? x0 : -INFINITY;
      x1 = lane + 32 <= jmax ? x1 : -INFINITY;
      float m = fmaxf(x0, x1);  // finite: key 0 is always in the chunk
      for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const float e0 = __expf(x0 - m), e1 = __expf(x1 - m);
      float l = e0 + e1;
      for (int o = 16; o; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
      ps[lane * GB + g] = e0;
      ps[(lane + 32) * GB + g] = e1;
      if (lane == 0) {
        st[g * 4 + 0] = m;
        st[g * 4 + 1] = l;
        // the chunk's fusion logit: its landmark logit, or for the own chunk
        // the log-sum-exp of its causal token logits
        st[g * 4 + 2] = (c == own) ? m + __logf(l) : ent_l[(i - i0) * GB + g];
      }
    }
    __syncthreads();
    // ---- P V over this thread's key slice, every head
    {
      const unsigned char *vb = smem + Lay::vs + buf * kC * Lay::kRow + pcol * 2 * (int)sizeof(T);
      float2 oa[GP], ob[GP];
#pragma unroll
      for (int gp = 0; gp < GP; ++gp) oa[gp] = ob[gp] = make_float2(0.0f, 0.0f);
      const int jlo = ksl * KPS, jend = min(jlo + KPS, jmax + 1);
#pragma unroll 4
      for (int j = jlo; j < jend; ++j) {
        float v0, v1;
        if constexpr (sizeof(T) == 2) {
          const uint32_t w = *reinterpret_cast<const uint32_t *>(vb + j * Lay::kRow);
          v0 = __uint_as_float(w << 16);
          v1 = __uint_as_float(w & 0xFFFF0000u);
        } else {
          const float2 w = *reinterpret_cast<const float2 *>(vb + j * Lay::kRow);
          v0 = w.x;
          v1 = w.y;
        }
        const float *pj = ps + j * GB;
        if constexpr (GB == 1) {
          oa[0].x = fmaf(pj[0], v0, oa[0].x);
          ob[0].x = fmaf(pj[0], v1, ob[0].x);
        } else {
#pragma unroll
          for (int gp = 0; gp < GP; ++gp) {
            const float2 pp = *reinterpret_cast<const float2 *>(pj + 2 * gp);
            oa[gp] = __ffma2_rn(pp, make_float2(v0, v0), oa[gp]);
            ob[gp] = __ffma2_rn(pp, make_float2(v1, v1), ob[gp]);
          }
        }
      }
      // acc_g = acc_g exp(M_old - M_new) + exp(logit - M_new) / l * o_g
      float so[GB], sn[GB];
#pragma unroll
      for (int g = 0; g < GB; ++g) {
        so[g] = 1.0f;
        sn[g] = 0.0f;
        if (g < G && ((mask >> g) & 1u)) {
          const float lg = st[g * 4 + 2], l = st[g * 4 + 1];
          const float mn = fmaxf(Mr[g], lg);
          so[g] = __expf(Mr[g] - mn);
          const float e = __expf(lg - mn);
          sn[g] = e / l;
          Lr[g] = Lr[g] * so[g] + e;
          Mr[g] = mn;
        }
      }
      if constexpr (GB == 1) {
        acc_a[0].x = acc_a[0].x * so[0] + sn[0] * oa[0].x;
        acc_b[0].x = acc_b[0].x * so[0] + sn[0] * ob[0].x;
      } else {
#pragma unroll
        for (int gp = 0; gp < GP; ++gp) {
          const float2 s_o = make_float2(so[2 * gp], so[2 * gp + 1]);
          const float2 s_n = make_float2(sn[2 * gp], sn[2 * gp + 1]);
          acc_a[gp] = __ffma2_rn(acc_a[gp], s_o, __fmul2_rn(s_n, oa[gp]));
          acc_b[gp] = __ffma2_rn(acc_b[gp], s_o, __fmul2_rn(s_n, ob[gp]));
        }
      }
    }
    __syncthreads();  // the buffer, xs, ps and st are reused
  }
  __syncthreads();  // every copy has landed (also on the timeout path)
  // ---- sum the key slices; partial record per (bk, qi, g): [M, L, acc[D]]
  float *red = reinterpret_cast<float *>(smem + Lay::ks);  // [KS][GB][D]
#pragma unroll
  for (int gp = 0; gp < GP; ++gp) {
#pragma unroll
    for (int u = 0; u < (GB == 1 ? 1 : 2); ++u) {
      const int g = 2 * gp + u;
      const float a = u ? acc_a[gp].y : acc_a[gp].x, bb = u ? acc_b[gp].y : acc_b[gp].x;
      *reinterpret_cast<float2 *>(red + (ksl * GB + g) * D + 2 * pcol) = make_float2(a, bb);
    }
  }
  __syncthreads();
  const size_t rec = 2 + D;
  for (int i = tid; i < G * D; i += kAttnThreads) {
    const int g = i / D, e = i % D;
    float sum = 0.0f;
#pragma unroll
    for (int k2 = 0; k2 < KS; ++k2) sum += red[(k2 * GB + g) * D + e];
    part[(((size_t)bk * ds.Q + qi) * G + g) * rec + 2 + e] = sum;
  }
  if (tid < G) {
    float mo = 0.0f, lo = 0.0f;
#pragma unroll
    for (int g = 0; g < GB; ++g)
      if (g == tid) { mo = Mr[g]; lo = Lr[g]; }
    float *r = part + (((size_t)bk * ds.Q + qi) * G + tid) * rec;
    r[0] = mo;
    r[1] = lo;
  }
  if (tid == 0 && *abort_flag) report(err, DEV_TIMEOUT);
}

// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(DecodeSpec ds,
                                                           const float *__restrict__ part,
                                                           T *__restrict__ out,
                                                           float *__restrict__ lse) {
  const int G = ds.Hq / ds.Hkv;
  const int h = blockIdx.x;  // b*Hq + hq
  const int b = h / ds.Hq, hq = h % ds.Hq;
  const int bk = b * ds.Hkv + hq / G, g = hq % G;
  const size_t rec = 2 + D, stride = (size_t)G * rec;  // partial s of the head at r0 + s * stride
  __shared__ float m_s;
  grid_dep_wait();  // the chunk attention's partials
  const float *r0 = part + ((size_t)bk * ds.Q * G + g) * rec;
  // the partials' maximum: one load per lane of the first warp
  if (threadIdx.x < 32) {
    float m = -INFINITY;
    for (int s = threadIdx.x; s < ds.Q; s += 32) m = fmaxf(m, r0[s * stride]);
#pragma unroll
    for (int o2 = 16; o2; o2 >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o2));
    if (threadIdx.x == 0) m_s = m;
  }
  __syncthreads();
  const float M = m_s;
  // one pass over the partials in order, their loads independent of each other
  float L = 0.0f, o = 0.0f;
#pragma unroll 8
  for (int s = 0; s < ds.Q; ++s) {
    const float *r = r0 + s * stride;
    const float m = r[0];
    if (m == -INFINITY) continue;
    const float w = __expf(m - M);
    L += w * r[1];
    o += w * r[2 + threadIdx.x];
  }
  out[(size_t)h * D + threadIdx.x] = from_f<T>(o / L);
  if (threadIdx.x == 0) lse[h] = M + __logf(L);
}

}  // namespace

DecodeSpec decode_spec(int B, int Hq, int Hkv, int N, int d, int topk, float scale) {
  DecodeSpec ds{};
  ds.B = B;
  ds.Hq = Hq;
  ds.Hkv = Hkv;
  ds.N = N;
  ds.d = d;
  ds.topk = topk;
  ds.scale = scale;
  ds.own = (N - 1) / kC;
  ds.nlmk = N / kC;
  ds.n_c = ds.own;  // completed chunks of the query at N-1 (all of them have a landmark)
  ds.P = (ds.n_c + kGemvThreads - 1) / kGemvThreads;
  ds.nwords = ((N + kC - 1) / kC + 31) / 32;
  const int G = Hq / Hkv;
  ds.ucap = G * topk + 1;
  ds.Q = (ds.ucap + kChunksPerCta - 1) / kChunksPerCta;
  return ds;
}

// workspace carve-up (256-byte aligned pieces)
static size_t al(size_t x) { return (x + 255) & ~size_t(255); }
size_t decode_workspace_bytes(const DecodeSpec &ds) {
  const int G = ds.Hq / ds.Hkv;
  const size_t BK = (size_t)ds.B * ds.Hkv;
  size_t n = 256;                                          // error word
  n += al(BK * ds.ucap * sizeof(int32_t));                 // u_c
  n += al(BK * ds.ucap * sizeof(uint32_t));                // u_mask
  n += al(BK * ds.ucap * G * sizeof(float));               // u_logit
  n += al(BK * sizeof(int32_t));                           // u_count
  // the landmark logits [B*Hq][n_c] are dead before the attention partials
  // [B*Hkv][Q][G][2+d] are written: one region holds both
  n += al(std::max(BK * G * (size_t)ds.n_c, BK * ds.Q * G * (size_t)(2 + ds.d)) * sizeof(float));
  return n;
}

size_t decode_max_g() { return kMaxG; }

// A launch that may overlap the end of the kernel before it in the stream
// (programmatic stream serialization): the kernel's grid_dep_wait() orders
// its reads of that kernel's results.  dep = false: an ordinary launch.
template <typename... KArgs, typename... Args>
static cudaError_t launch_dep(bool dep, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args &&...args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = dep ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// The five launches of one decode step; pages.table == nullptr: dense caches.
// Each launch after the first may start while the one before it finishes; the
// first (the landmark pass, or the top-k when there is none) is an ordinary
// launch, so the step's inputs are complete before any of its kernels runs.
static cudaError_t decode_run(const DecodeSpec &ds, bool bf16, const void *q, const void *k,
                              const void *v, const PagedKV &pages, const void *lmk, int32_t *sel,
                              float *w, float *lse_lmk, void *out, float *lse, void *ws,
                              uint32_t *err, cudaStream_t st, int *launches) {
  const int G = ds.Hq / ds.Hkv;
  const size_t BK = (size_t)ds.B * ds.Hkv;
  unsigned char *p = static_cast<unsigned char *>(ws) + 256;
  auto take = [&](size_t bytes) {
    unsigned char *r = p;
    p += al(bytes);
    return r;
  };
  int32_t *u_c = reinterpret_cast<int32_t *>(take(BK * ds.ucap * 4));
  uint32_t *u_mask = reinterpret_cast<uint32_t *>(take(BK * ds.ucap * 4));
  float *u_logit = reinterpret_cast<float *>(take(BK * ds.ucap * G * 4));
  int32_t *u_count = reinterpret_cast<int32_t *>(take(BK * 4));
  float *part = reinterpret_cast<float *>(
      take(std::max(BK * G * (size_t)ds.n_c, BK * ds.Q * G * (size_t)(2 + ds.d)) * 4));
  float *scores = part;  // landmark logits, consumed before the partials are written
  cudaError_t e;

  if (ds.P > 0 && bf16 && G <= kTcN) {
    CUtensorMap tl;
    if ((e = make_tmap_bf16(&tl, lmk, (uint64_t)BK * ds.nlmk, ds.d, kTcRows)) != cudaSuccess) return e;
    const int ntiles = (ds.n_c + kTcRows - 1) / kTcRows;
    const dim3 grid((unsigned)std::min(ntiles, kTcTilesPerCta), (unsigned)BK);
#define HILS_GEMV_TC(DD)                                                                        \
  do {                                                                                          \
    auto kern = decode_gemv_tc_kernel<DD>;                                                      \
    const size_t smem = GemvTcLayout<DD>::total;                                                \
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess) return e; \
    kern<<<grid, 192, smem, st>>>(tl, ds, (const __nv_bfloat16 *)q, scores, err);               \
  } while (0)
    if (ds.d == 64) HILS_GEMV_TC(64); else HILS_GEMV_TC(128);
#undef HILS_GEMV_TC
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    ++*launches;
  } else if (ds.P > 0) {
#define HILS_GEMV(T, DD) \
  decode_gemv_kernel<T, DD><<<dim3(ds.P, (unsigned)BK), kGemvThreads, 0, st>>>(ds, (const T *)q, (const T *)lmk, scores)
    if (bf16) { if (ds.d == 64) HILS_GEMV(__nv_bfloat16, 64); else HILS_GEMV(__nv_bfloat16, 128); }
    else { if (ds.d == 64) HILS_GEMV(float, 64); else HILS_GEMV(float, 128); }
#undef HILS_GEMV
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    ++*launches;
  }
  {
    // stage the head's logits in shared memory when they fit
    const size_t tsmem = (size_t)ds.n_c * sizeof(float);
    const int staged = tsmem <= 160 * 1024 ? 1 : 0;
    if (staged && (e = cudaFuncSetAttribute(decode_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tsmem)) != cudaSuccess) return e;
    if ((e = launch_dep(ds.P > 0, decode_topk_kernel, dim3((unsigned)(ds.B * ds.Hq)), dim3(kTkThreads),
                        staged ? tsmem : 0, st, ds, (const float *)scores, sel, w, lse_lmk, staged)) != cudaSuccess)
      return e;
  }
  ++*launches;
  {
    const size_t smem = (size_t)G * ds.topk * 8 + (size_t)ds.nwords * 8;
    if ((e = cudaFuncSetAttribute(decode_union_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess) return e;
    if ((e = launch_dep(true, decode_union_kernel, dim3((unsigned)BK), dim3(256), smem, st, ds,
                        (const int32_t *)sel, (const float *)w, u_c, u_mask, u_logit, u_count)) != cudaSuccess)
      return e;
    ++*launches;
  }
  {
    // K through a 2-D tensor map: the dense cache [B*Hkv*N rows][d], or the
    // page pool [num_pages*Hkv*64 rows][d]
    const uint64_t krows = pages.table ? (uint64_t)pages.num_pages * ds.Hkv * kC : (uint64_t)BK * ds.N;
    if (krows >= (1ull << 31)) return cudaErrorInvalidValue;  // tensor-map rows are int32
    CUtensorMap tk;
    if ((e = bf16 ? make_tmap_bf16(&tk, k, krows, ds.d, kC) : make_tmap_f32(&tk, k, krows, ds.d, kC)) != cudaSuccess)
      return e;
#define HILS_ATTN(T, DD, GG)                                                                    \
  do {                                                                                          \
    auto kern = decode_attn_kernel<T, DD, GG>;                                                  \
    const size_t smem = DecAttnLayout<T, DD, GG>::total;                                        \
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess) return e; \
    if ((e = launch_dep(true, kern, dim3(ds.Q, (unsigned)BK), dim3(kAttnThreads), smem, st, tk, ds,   \
                        (const T *)q, (const T *)k, (const T *)v, pages, (const int32_t *)u_c,   \
                        (const uint32_t *)u_mask, (const float *)u_logit,                        \
                        (const int32_t *)u_count, part, err)) != cudaSuccess)                    \
      return e;                                                                                 \
  } while (0)
#define HILS_ATTN_G(T, DD)                                                                      \
  do {                                                                                          \
    if (G <= 1) HILS_ATTN(T, DD, 1);                                                            \
    else if (G <= 2) HILS_ATTN(T, DD, 2);                                                       \
    else if (G <= 4) HILS_ATTN(T, DD, 4);                                                       \
    else HILS_ATTN(T, DD, 8);                                                                   \
  } while (0)
    if (bf16) { if (ds.d == 64) HILS_ATTN_G(__nv_bfloat16, 64); else HILS_ATTN_G(__nv_bfloat16, 128); }
    else { if (ds.d == 64) HILS_ATTN_G(float, 64); else HILS_ATTN_G(float, 128); }
#undef HILS_ATTN_G
#undef HILS_ATTN
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    ++*launches;
  }
  {
    const int nh = ds.B * ds.Hq;
#define HILS_COMB(T, DD)                                                                        \
  do {                                                                                          \
    if ((e = launch_dep(true, decode_combine_kernel<T, DD>, dim3((unsigned)nh), dim3(DD), 0, st, ds,    \
                        (const float *)part, (T *)out, lse)) != cudaSuccess)                     \
      return e;                                                                                 \
  } while (0)
    if (bf16) { if (ds.d == 64) HILS_COMB(__nv_bfloat16, 64); else HILS_COMB(__nv_bfloat16, 128); }
    else { if (ds.d == 64) HILS_COMB(float, 64); else HILS_COMB(float, 128); }
#undef HILS_COMB
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    ++*launches;
  }
  return cudaSuccess;
}

cudaError_t decode_fwd(const DecodeSpec &ds, bool bf16, const void *q, const void *k,
                       const void *v, const void *lmk, int32_t *sel, float *w, float *lse_lmk,
                       void *out, float *lse, void *ws, uint32_t *err, cudaStream_t st,
                       int *launches) {
  return decode_run(ds, bf16, q, k, v, PagedKV{nullptr, 0, 0}, lmk, sel, w, lse_lmk, out, lse, ws,
                    err, st, launches);
}

cudaError_t decode_fwd_paged(const DecodeSpec &ds, bool bf16, const void *q, const void *k_pages,
                             const void *v_pages, const PagedKV &pages, const void *lmk,
                             int32_t *sel, float *w, float *lse_lmk, void *out, float *lse,
                             void *ws, uint32_t *err, cudaStream_t st, int *launches) {
  return decode_run(ds, bf16, q, k_pages, v_pages, pages, lmk, sel, w, lse_lmk, out, lse, ws, err,
                    st, launches);
}

}  // namespace hils
