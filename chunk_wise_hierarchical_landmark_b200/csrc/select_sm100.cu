// Landmark scoring, inter-chunk normaliser and top-k chunk selection on the
// 5th-generation tensor cores (model card "HiLS-Attention", section "What
// HiLS-Attention is"; molayo1419.me, "Core idea" step 1): for every query row
// t the logits s_c = scale * <q_t, lmk_c> of its completed chunks c < t/C,
// their log-sum-exp, and the k best by (s desc, c asc).
//
// One CTA = 128 query rows of one (b, hq); two CTAs share an SM.  6 warps:
//   warp 0     TMA producer: the Q tile into the landmark ring (staging), then
//              64-landmark tiles of the row block's KV head into a 2-stage ring;
//   warp 1     TMEM owner, MMA issuer: S = Q Lmk^T (128 x 64 fp32) into one of
//              two TMEM buffers, with Q as the A operand in tensor memory;
//   warps 2-5  one thread per row (TMEM lane): copy the row's q into tensor
//              memory, then per 32-candidate block an online log-sum-exp (base
//              2) and the row's best k keys in shared memory (8 groups of 8
//              slots, group minima in registers).  A block whose best score
//              cannot enter is skipped; the first k candidates are appended
//              without search; qualifying candidates later are staged in shared
//              memory and inserted one per lane per step, so the 32 rows of a
//              warp insert together.  Chunks arrive in ascending order, so a
//              later chunk never wins a tie.
// The candidate scores never leave the chip.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace hils {
namespace {

using namespace sm100;

constexpr int kRows = 128;
constexpr int kTile = 64;     // landmarks per MMA tile (UMMA N)
constexpr int kStages = 2;
constexpr int kThreads = 192;
constexpr int kMaxK = 64;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <int D>
struct SelLayout {
  static constexpr int kQBytes = kRows * D * 2;
  static constexpr int kLBytes = kTile * D * 2;
  static_assert(kStages * kLBytes == kQBytes, "the landmark ring stages the Q tile");
  static constexpr int l0 = 0;                               // landmark ring / Q staging
  static constexpr int heap = l0 + kStages * kLBytes;        // [kMaxK][128] uint64 slots
  static constexpr int stage = heap + kMaxK * kRows * 8;     // [32][128] fp32 candidate staging
  static constexpr int bars = stage + 32 * kRows * 4;
  static constexpr int misc = bars + 16 * 8;
  static constexpr int total = misc + 32;
  // TMEM columns: Q [0, D/2) as bf16 pairs, S0 [64, 128), S1 [128, 192)
  static constexpr uint32_t kQCol = 0, kSCol = 64, kTmemCols = 256;
};

struct SelBars {
  uint64_t q_smem, q_tmem, l_full[kStages], l_empty[kStages], s_full[2], s_empty[2], done;
};

// Per-row top-k: kMaxK key slots in shared memory (slot i of the row at
// h[i * 128]) in 8 groups of 8, each group's minimum (key and position) kept
// in registers.  Replacing the overall minimum rescans one group (8
// independent loads, tree minimum) instead of walking a heap.  Slots >= K
// count as +inf.
struct TopK {
  uint64_t gmin[8];
  uint32_t gpos;  // 3 bits per group: position of the group's minimum
  uint64_t mn;    // overall minimum (the entry a better key replaces)
  int mg;         // its group
  int cnt;        // filled slots
  float thr;      // score of mn once all K slots are filled, -inf before

  __device__ __forceinline__ void rescan(const uint64_t *h, int g, int K) {
    uint64_t x[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int slot = g * 8 + i;
      x[i] = slot < K ? h[slot * kRows] : ~0ull;
    }
    // tree minimum with positions
    const uint64_t m01 = x[0] <= x[1] ? x[0] : x[1];
    const uint32_t p01 = x[0] <= x[1] ? 0u : 1u;
    const uint64_t m23 = x[2] <= x[3] ? x[2] : x[3];
    const uint32_t p23 = x[2] <= x[3] ? 2u : 3u;
    const uint64_t m45 = x[4] <= x[5] ? x[4] : x[5];
    const uint32_t p45 = x[4] <= x[5] ? 4u : 5u;
    const uint64_t m67 = x[6] <= x[7] ? x[6] : x[7];
    const uint32_t p67 = x[6] <= x[7] ? 6u : 7u;
    const uint64_t ma = m01 <= m23 ? m01 : m23;
    const uint32_t pa = m01 <= m23 ? p01 : p23;
    const uint64_t mb = m45 <= m67 ? m45 : m67;
    const uint32_t pb = m45 <= m67 ? p45 : p67;
    const uint64_t m = ma <= mb ? ma : mb;
    const uint32_t pos = ma <= mb ? pa : pb;
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (i == g) gmin[i] = m;
    gpos = (gpos & ~(7u << (3 * g))) | (pos << (3 * g));
  }
  __device__ __forceinline__ void overall() {
    const uint64_t a0 = gmin[0] <= gmin[1] ? gmin[0] : gmin[1];
    const int i0 = gmin[0] <= gmin[1] ? 0 : 1;
    const uint64_t a1 = gmin[2] <= gmin[3] ? gmin[2] : gmin[3];
    const int i1 = gmin[2] <= gmin[3] ? 2 : 3;
    const uint64_t a2 = gmin[4] <= gmin[5] ? gmin[4] : gmin[5];
    const int i2 = gmin[4] <= gmin[5] ? 4 : 5;
    const uint64_t a3 = gmin[6] <= gmin[7] ? gmin[6] : gmin[7];
    const int i3 = gmin[6] <= gmin[7] ? 6 : 7;
    const uint64_t b0 = a0 <= a1 ? a0 : a1;
    const int j0 = a0 <= a1 ? i0 : i1;
    const uint64_t b1 = a2 <= a3 ? a2 : a3;
    const int j1 = a2 <= a3 ? i2 : i3;
    mn = b0 <= b1 ? b0 : b1;
    mg = b0 <= b1 ? j0 : j1;
    thr = key_score(mn);
  }
  __device__ __forceinline__ void build(const uint64_t *h, int K) {
#pragma unroll
    for (int g = 0; g < 8; ++g) rescan(h, g, K);
    overall();
  }
  // replace the overall minimum with `key` (the caller checked key > mn)
  __device__ __forceinline__ void replace(uint64_t *h, uint64_t key, int K) {
    const int slot = mg * 8 + ((gpos >> (3 * mg)) & 7u);
    h[slot * kRows] = key;
    rescan(h, mg, K);
    overall();
  }
};

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
    select_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_l, RowSpec rs,
                        int32_t *__restrict__ sel, float *__restrict__ chunk_w,
                        float *__restrict__ lse_lmk, uint32_t *__restrict__ err) {
  using Lay = SelLayout<D>;
  // The 128-byte-swizzled tiles need a 1024-byte aligned base; the dynamic
  // shared window starts there (there is no static shared memory), which the
  // kernel checks rather than assumes.
  extern __shared__ __align__(1024) unsigned char smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) report(err, DEV_BAD_INDEX);
    return;
  }
  SelBars *bars = reinterpret_cast<SelBars *>(smem + Lay::bars);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Lay::misc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Lay::misc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int b = bh / rs.Hq, hq = bh % rs.Hq, hkv = hq / (rs.Hq / rs.Hkv);
  const int ntiles_rows = (rs.L + kRows - 1) / kRows;
  const int t0 = (ntiles_rows - 1 - blockIdx.x) * kRows;  // heaviest tiles first
  const int L = rs.L, K = rs.topk, C = rs.C;
  const int nlmk = L / C;
  const int t_last = min(t0 + kRows, L) - 1;
  const int n_cand = min(t_last / C, nlmk);  // candidates of the tile's last row
  const int n_ltiles = (n_cand + kTile - 1) / kTile;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_smem, 1);
    mbar_init(&bars->q_tmem, kRows);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->l_full[s], 1);
      mbar_init(&bars->l_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->s_empty[i], kRows);
    }
    mbar_init(&bars->done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_l);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Lay::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t q_tmem = tmem + Lay::kQCol;
  const uint32_t s_tmem[2] = {tmem + Lay::kSCol, tmem + Lay::kSCol + kTile};
  const int lrow0 = (b * rs.Hkv + hkv) * nlmk;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n_ltiles > 0) {
      mbar_expect_tx(&bars->q_smem, Lay::kQBytes);
      for (int kb = 0; kb < D / 64; ++kb)
        tma_load_2d(smem + Lay::l0 + kb * kRows * 128, &tm_q, &bars->q_smem, kb * 64, bh * L + t0);
      // the ring holds the Q tile until the row threads have moved it to TMEM
      const bool ok = mbar_wait(&bars->q_tmem, 0, abort_flag);
      int issued = 0;
      for (int i = 0; ok && i < n_ltiles; ++i) {
        const int s = i % kStages;
        if (i >= kStages && !mbar_wait(&bars->l_empty[s], ((i / kStages) - 1) & 1, abort_flag))
          break;
        mbar_expect_tx(&bars->l_full[s], Lay::kLBytes);
        unsigned char *ls = smem + Lay::l0 + s * Lay::kLBytes;
        for (int kb = 0; kb < D / 64; ++kb)
          tma_load_2d(ls + kb * kTile * 128, &tm_l, &bars->l_full[s], kb * 64, lrow0 + i * kTile);
        ++issued;
      }
      for (int i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
        mbar_wait_bounded(&bars->l_full[i % kStages], (i / kStages) & 1);
      mbar_wait_bounded(&bars->q_smem, 0);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_ltiles > 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kRows, kTile, false, false);
      const bool ok = mbar_wait(&bars->q_tmem, 0, abort_flag);
      tc_fence_after();
      for (int i = 0; ok && i < n_ltiles; ++i) {
        const int s = i % kStages, sb = i & 1;
        if (!mbar_wait(&bars->l_full[s], (i / kStages) & 1, abort_flag)) break;
        if (i >= 2 && !mbar_wait(&bars->s_empty[sb], ((i >> 1) - 1) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t l_addr = smem_u32(smem + Lay::l0 + s * Lay::kLBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int kb = kk >> 2, kw = kk & 3;
          const uint64_t bd = smem_desc_sw128(l_addr + kb * kTile * 128 + kw * 32, 16, 1024);
          mma_bf16_ts(s_tmem[sb], q_tmem + kk * 8, bd, idesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars->s_full[sb]);
        mma_commit(&bars->l_empty[s]);
      }
      mma_commit(&bars->done);
      mbar_wait_bounded(&bars->done, 0);
    }
  } else {
    // ---------------------------------------------------------- row threads
    const int r = 32 * (warp & 3) + lane;
    const int t = t0 + r;
    const bool valid = t < L;
    const int n_c = valid ? min(t / C, nlmk) : 0;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    uint64_t *slots = reinterpret_cast<uint64_t *>(smem + Lay::heap) + r;
    float *stage = reinterpret_cast<float *>(smem + Lay::stage) + r;
    const float c2 = rs.scale * kLog2e;
    const float sc = rs.scale;
    const bool want_lse = lse_lmk != nullptr;
    float m2 = -INFINITY, l = 0.0f;
    TopK tk;
    tk.cnt = 0;
    tk.thr = -INFINITY;
    tk.gpos = 0;
    tk.mn = 0;
    tk.mg = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) tk.gmin[i] = ~0ull;
    bool ok = true;
    if (n_ltiles > 0) {
      // q row -> tensor memory (A operand of the scoring MMA): the row's
      // 128-byte lines of the swizzled staging tile, two bf16 per column
      ok = mbar_wait(&bars->q_smem, 0, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb) {
          uint32_t w[32];
          const unsigned char *line = smem + Lay::l0 + kb * kRows * 128 + r * 128;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint4 v4 = *reinterpret_cast<const uint4 *>(line + ((j ^ (r & 7)) << 4));
            w[4 * j] = v4.x;
            w[4 * j + 1] = v4.y;
            w[4 * j + 2] = v4.z;
            w[4 * j + 3] = v4.w;
          }
          tmem_st32(q_tmem + lane_off + kb * 32, w);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(&bars->q_tmem);
    }
    for (int i = 0; ok && i < n_ltiles; ++i) {
      const int sb = i & 1;
      ok = mbar_wait(&bars->s_full[sb], (i >> 1) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      float a2[2][32];
      tmem_ld32(s_tmem[sb] + lane_off, a2[0]);
      tmem_ld32(s_tmem[sb] + lane_off + 32, a2[1]);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bars->s_empty[sb]);
#pragma unroll
      for (int blk = 0; blk < 2; ++blk) {
        float(&a)[32] = a2[blk];
        const int cb = i * kTile + blk * 32;
        const int nv = max(0, min(32, n_c - cb));
        if (nv < 32) {
#pragma unroll
          for (int j = 0; j < 32; ++j) a[j] = j < nv ? a[j] : -INFINITY;
        }
        // block maximum (tree)
        float mx[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) mx[j] = fmaxf(a[j], a[j + 16]);
#pragma unroll
        for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
          for (int j = 0; j < w; ++j) mx[j] = fmaxf(mx[j], mx[j + w]);
        const float bm = mx[0];
        if (want_lse && nv > 0) {
          const float bm2 = bm * c2;
          if (bm2 > m2) {
            l *= ex2_approx(m2 - bm2);
            m2 = bm2;
          }
          float ps[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
          for (int j = 0; j < 32; ++j) ps[j & 3] += ex2_approx(fmaf(a[j], c2, -m2));
          l += (ps[0] + ps[1]) + (ps[2] + ps[3]);
        }
        const bool fill = nv > 0 && tk.cnt + nv <= K;
        if (fill) {
          // fill phase: every candidate is kept; append without search
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < nv) slots[(tk.cnt + j) * kRows] = sel_key(a[j] * sc, cb + j);
          tk.cnt += nv;
          if (tk.cnt == K) tk.build(slots, K);
        }
        // candidates that may enter the top-k (the vote below is warp-wide:
        // every lane reaches it, filling lanes with an empty mask)
        uint32_t mask = 0;
        if (!fill && nv > 0 && (tk.cnt < K || bm * sc > tk.thr)) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            mask |= (j < nv && (tk.cnt < K || a[j] * sc > tk.thr)) ? (1u << j) : 0u;
        }
        if (__any_sync(0xffffffffu, mask != 0)) {
          if (mask) {
#pragma unroll
            for (int j = 0; j < 32; ++j) stage[j * kRows] = a[j];
          }
          // one candidate per lane per iteration: the lanes insert together
          while (__any_sync(0xffffffffu, mask != 0)) {
            if (mask) {
              const int j = __ffs(mask) - 1;
              mask &= mask - 1;
              const float s = stage[j * kRows] * sc;
              const uint64_t key = sel_key(s, cb + j);
              if (tk.cnt < K) {
                slots[tk.cnt * kRows] = key;
                if (++tk.cnt == K) tk.build(slots, K);
              } else if (s > tk.thr) {
                tk.replace(slots, key, K);
              }
            }
          }
        }
      }
    }
    if (__all_sync(0xffffffffu, ok) && valid) {
      // ascending chunk order: insertion sort of the kept keys by chunk id
      const int cnt = tk.cnt;
      for (int i = 1; i < cnt; ++i) {
        const uint64_t x = slots[i * kRows];
        const int cx = key_chunk(x);
        int j = i - 1;
        while (j >= 0 && key_chunk(slots[j * kRows]) > cx) {
          slots[(j + 1) * kRows] = slots[j * kRows];
          --j;
        }
        slots[(j + 1) * kRows] = x;
      }
      const size_t row = (size_t)bh * L + t;
      int32_t *srow = sel + row * K;
      float *wrow = chunk_w + row * K;
      if ((K & 3) == 0) {
        for (int i = 0; i < K; i += 4) {
          int4 si;
          float4 wi;
          int *sp = &si.x;
          float *wp = &wi.x;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const bool have = i + u < cnt;
            const uint64_t x = have ? slots[(i + u) * kRows] : 0;
            sp[u] = have ? key_chunk(x) : -1;
            wp[u] = have ? key_score(x) : -INFINITY;
          }
          *reinterpret_cast<int4 *>(srow + i) = si;
          *reinterpret_cast<float4 *>(wrow + i) = wi;
        }
      } else {
        for (int i = 0; i < K; ++i) {
          const bool have = i < cnt;
          const uint64_t x = have ? slots[i * kRows] : 0;
          srow[i] = have ? key_chunk(x) : -1;
          wrow[i] = have ? key_score(x) : -INFINITY;
        }
      }
      if (want_lse) lse_lmk[row] = n_c > 0 ? (m2 + __log2f(l)) * kLn2 : -INFINITY;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) report(err, DEV_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Lay::kTmemCols);
  }
}

}  // namespace

cudaError_t select_sm100(const RowSpec &rs, const void *q, const void *lmk, int32_t *sel,
                         float *w, float *lse_lmk, uint32_t *err, cudaStream_t st) {
  CUtensorMap tq, tl;
  cudaError_t e;
  const int nlmk = rs.L / rs.C;
  const uint64_t qrows = (uint64_t)rs.B * rs.Hq * rs.L;
  const uint64_t lrows = (uint64_t)rs.B * rs.Hkv * (nlmk > 0 ? nlmk : 1);
  if ((e = make_tmap_bf16(&tq, q, qrows, rs.d, kRows)) != cudaSuccess) return e;
  // with no complete chunk the landmark map is never read; point it at q
  if ((e = make_tmap_bf16(&tl, nlmk > 0 ? lmk : q, lrows, rs.d, kTile)) != cudaSuccess) return e;
  dim3 grid((rs.L + kRows - 1) / kRows, rs.B * rs.Hq);
  if (rs.d == 64) {
    const size_t smem = SelLayout<64>::total;
    auto kern = select_sm100_kernel<64>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess) return e;
    kern<<<grid, kThreads, smem, st>>>(tq, tl, rs, sel, w, lse_lmk, err);
  } else {
    const size_t smem = SelLayout<128>::total;
    auto kern = select_sm100_kernel<128>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess) return e;
    kern<<<grid, kThreads, smem, st>>>(tq, tl, rs, sel, w, lse_lmk, err);
  }
  return cudaGetLastError();
}

}  // namespace hils
