// Landmark scoring, inter-chunk normaliser and top-k chunk selection on the
// 5th-generation tensor cores (model card "HiLS-Attention", section "What
// HiLS-Attention is"; molayo1419.me, "Core idea" step 1): for every query row
// t the logits s_c = scale * <q_t, lmk_c> of its completed chunks c < t/C,
// their log-sum-exp, and the k best by (s desc, c asc).
//
// One CTA = 128 query rows of one (b, hq); 6 warps:
//   warp 0     TMA producer: the Q tile once, then 128-landmark tiles of the
//              row block's KV head into a 3-stage ring;
//   warp 1     TMEM owner, MMA issuer: S = Q Lmk^T (128 x 128 fp32) into one of
//              two TMEM buffers;
//   warps 2-5  one thread per row: block-wise online log-sum-exp and a binary
//              min-heap of the row's best k keys in shared memory.  A 32-wide
//              block of candidates is skipped whole when its best score cannot
//              enter the heap (chunks arrive in ascending order, so a later
//              chunk never wins a tie).
// The candidate scores never leave the chip.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace hils {
namespace {

using namespace sm100;

constexpr int kRows = 128;
constexpr int kTile = 128;    // landmarks per MMA tile (UMMA N)
constexpr int kStages = 3;
constexpr int kThreads = 192;
constexpr int kMaxK = 64;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <int D>
struct SelLayout {
  static constexpr int kQBytes = kRows * D * 2;
  static constexpr int kLBytes = kTile * D * 2;
  static constexpr int q = 0;
  static constexpr int l0 = q + kQBytes;
  static constexpr int heap = l0 + kStages * kLBytes;      // [kMaxK][128] uint64
  static constexpr int bars = heap + kMaxK * kRows * 8;
  static constexpr int misc = bars + 16 * 8;
  static constexpr int total = misc + 64;
  static constexpr uint32_t kTmemCols = 256;  // S0 [0,128), S1 [128,256)
};

struct SelBars {
  uint64_t q, l_full[kStages], l_empty[kStages], s_full[2], s_empty[2], done;
};

// Per-row top-k state: a binary min-heap of selection keys in shared memory
// (entry i of the row at h[i * 128]); `thr` is the root's score once full.
struct HeapState {
  int cnt;
  float thr;
};

// Insert `key` (the caller checked that it qualifies).  Kept out of line: it
// runs for a small fraction of the candidates.
__device__ __noinline__ HeapState heap_insert(uint64_t *h, HeapState st, int K, uint64_t key) {
  if (st.cnt < K) {  // sift up from the end
    int i = st.cnt;
    while (i > 0) {
      const int p = (i - 1) >> 1;
      const uint64_t kp = h[p * kRows];
      if (kp <= key) break;
      h[i * kRows] = kp;
      i = p;
    }
    h[i * kRows] = key;
    ++st.cnt;
  } else {  // replace the root and sift down
    int i = 0;
    while (true) {
      int c = 2 * i + 1;
      if (c >= K) break;
      uint64_t kc = h[c * kRows];
      if (c + 1 < K) {
        const uint64_t kr = h[(c + 1) * kRows];
        if (kr < kc) { kc = kr; ++c; }
      }
      if (key <= kc) break;
      h[i * kRows] = kc;
      i = c;
    }
    h[i * kRows] = key;
  }
  if (st.cnt == K) st.thr = key_score(h[0]);
  return st;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    select_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_l, RowSpec rs,
                        int32_t *__restrict__ sel, float *__restrict__ chunk_w,
                        float *__restrict__ lse_lmk, uint32_t *__restrict__ err) {
  using Lay = SelLayout<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
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
    mbar_init(&bars->q, 1);
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
  unsigned char *q_s = smem + Lay::q;
  const int lrow0 = (b * rs.Hkv + hkv) * nlmk;

  if (warp == 0) {
    if (lane == 0 && n_ltiles > 0) {
      mbar_expect_tx(&bars->q, Lay::kQBytes);
      for (int kb = 0; kb < D / 64; ++kb)
        tma_load_2d(q_s + kb * kRows * 128, &tm_q, &bars->q, kb * 64, bh * L + t0);
      int issued = 0;
      for (int i = 0; i < n_ltiles; ++i) {
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
      mbar_wait_bounded(&bars->q, 0);
    }
  } else if (warp == 1) {
    if (lane == 0 && n_ltiles > 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kRows, kTile, false, false);
      const uint32_t q_addr = smem_u32(q_s);
      bool ok = mbar_wait(&bars->q, 0, abort_flag);
      for (int i = 0; ok && i < n_ltiles; ++i) {
        const int s = i % kStages, sb = i & 1;
        if (!mbar_wait(&bars->l_full[s], (i / kStages) & 1, abort_flag)) break;
        if (i >= 2 && !mbar_wait(&bars->s_empty[sb], ((i >> 1) - 1) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t l_addr = smem_u32(smem + Lay::l0 + s * Lay::kLBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int kb = kk >> 2, kw = kk & 3;
          const uint64_t a = smem_desc_sw128(q_addr + kb * kRows * 128 + kw * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(l_addr + kb * kTile * 128 + kw * 32, 16, 1024);
          mma_bf16_ss(tmem + sb * kTile, a, bd, idesc, kk > 0 ? 1u : 0u);
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
    uint64_t *heap = reinterpret_cast<uint64_t *>(smem + Lay::heap) + r;
    const float c2 = rs.scale * kLog2e;
    const bool want_lse = lse_lmk != nullptr;
    float m2 = -INFINITY, l = 0.0f;
    HeapState hs{0, -INFINITY};
    bool ok = true;
    for (int i = 0; i < n_ltiles; ++i) {
      const int sb = i & 1;
      ok = mbar_wait(&bars->s_full[sb], (i >> 1) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
#pragma unroll 1
      for (int blk = 0; blk < kTile / 32; ++blk) {
        float a[32];
        __syncwarp();  // tcgen05.ld is warp-collective: reconverge after the divergent heap work
        tmem_ld32(tmem + sb * kTile + blk * 32 + lane_off, a);
        tmem_wait_ld();
        const int cb = i * kTile + blk * 32;
        if (cb >= n_c) continue;  // every candidate of this block is masked for this row
        const int nv = min(32, n_c - cb);
        if (nv < 32) {
#pragma unroll
          for (int j = 0; j < 32; ++j) a[j] = j < nv ? a[j] : -INFINITY;
        }
        float bm = a[0];
#pragma unroll
        for (int j = 1; j < 32; ++j) bm = fmaxf(bm, a[j]);
        if (want_lse) {
          const float bm2 = bm * c2;
          if (bm2 > m2) {
            l *= exp2f(m2 - bm2);
            m2 = bm2;
          }
          float part = 0.0f;
#pragma unroll
          for (int j = 0; j < 32; ++j) part += exp2f(fmaf(a[j], c2, -m2));
          l += part;
        }
        if (hs.cnt == K && bm * rs.scale <= hs.thr) continue;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float s = a[j] * rs.scale;  // masked candidates are -inf and never qualify
          if (j < nv && (hs.cnt < K || s > hs.thr)) hs = heap_insert(heap, hs, K, sel_key(s, cb + j));
        }
      }
      __syncwarp();
      tc_fence_before();
      mbar_arrive(&bars->s_empty[sb]);
    }
    if (__all_sync(0xffffffffu, ok) && valid) {
      // ascending chunk order: insertion sort of the chunk ids in place
      const int cnt = hs.cnt;
      for (int i = 1; i < cnt; ++i) {
        const uint64_t x = heap[i * kRows];
        const int cx = key_chunk(x);
        int j = i - 1;
        while (j >= 0 && key_chunk(heap[j * kRows]) > cx) {
          heap[(j + 1) * kRows] = heap[j * kRows];
          --j;
        }
        heap[(j + 1) * kRows] = x;
      }
      const size_t row = (size_t)bh * L + t;
      int32_t *srow = sel + row * K;
      float *wrow = chunk_w + row * K;
      for (int i = 0; i < K; ++i) {
        const bool have = i < cnt;
        const uint64_t x = have ? heap[i * kRows] : 0;
        srow[i] = have ? key_chunk(x) : -1;
        wrow[i] = have ? key_score(x) : -INFINITY;
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
    const size_t smem = SelLayout<64>::total + 1024;
    auto kern = select_sm100_kernel<64>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess) return e;
    kern<<<grid, kThreads, smem, st>>>(tq, tl, rs, sel, w, lse_lmk, err);
  } else {
    const size_t smem = SelLayout<128>::total + 1024;
    auto kern = select_sm100_kernel<128>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess) return e;
    kern<<<grid, kThreads, smem, st>>>(tq, tl, rs, sel, w, lse_lmk, err);
  }
  return cudaGetLastError();
}

}  // namespace hils
