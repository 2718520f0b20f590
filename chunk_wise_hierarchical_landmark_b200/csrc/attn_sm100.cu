// Intra-chunk attention + score-weighted fusion on the 5th-generation tensor
// cores (tcgen05, accumulators in tensor memory, operands staged by TMA).
//
// Method (molayo1419.me, "Core idea" step 2 and "Hardware-efficient kernel";
// aiweekly.co mechanism paragraph): each query attends, with an ordinary
// softmax, to each of its selected chunks and to its own chunk (causally);
// the per-chunk outputs are fused with weights softmax(chunk logits), the
// own chunk's logit being the log-sum-exp of its causal token logits.  A tile
// of 128 adjacent queries of one head loads the union of their chunks once.
//
// One CTA = one tile of 128 query rows (positions [t0, t0+128) of one
// (b, hq)); two CTAs share an SM (about 100 KB of shared memory and 256 TMEM
// columns each).  6 warps:
//   warp 0     TMA producer: Q tile once, then K_c / V_c of every union chunk
//              into a 2-stage ring;
//   warp 1     TMEM owner and MMA issuer (one thread): S = Q K_c^T into TMEM,
//              then O += P_c V_c reading P from tensor memory;
//   warps 2-5  one thread per row (TMEM lane): chunk softmax, P -> tensor
//              memory (bf16, two per column, over the chunk's own S), the
//              running sum of the rounded P, epilogue.
// S is double-buffered: while the rows turn S_j into P_j, S_{j+1} is ready
// in the other buffer, and S_{j+2} is computed into this one as soon as
// P_j·V_j has read P_j.
//
// Processing order: the tile's own chunks first (later one first), then the
// rest of the union ascending.  After its own chunk a row knows its largest
// fusion logit M = max(lse_own, max selected logit), so every chunk's
// probabilities are written directly against M:
//   P_j = exp(x_j - m_c) / l_c * exp(s_c - M)       (selected chunk c)
//   P_j = exp(x_j - M)                               (own chunk)
// and O = sum_c P_c V_c needs no rescaling.  P is rounded to bf16 for the
// tensor core; the output is normalised by the sum of the ROUNDED
// probabilities (accumulated in fp32 by the row threads from the bf16 values
// they store), so the weights applied to V sum to one: out = O / sum_j
// bf16(P_j).  lse stays the fp32 value M + log(sum_c exp(s_c - M)).
#include <cuda_bf16.h>

#include "common.cuh"
#include "hope.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace hils {
namespace {

using namespace sm100;

constexpr int kRows = 128;   // query rows per tile (UMMA M)
constexpr int kChunk = 64;   // keys per chunk (UMMA N of QK^T, K of PV)
constexpr int kStages = 2;   // K/V ring depth
constexpr int kThreads = 192;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <int D>
struct Layout {
  static constexpr int kQBytes = kRows * D * 2;
  static constexpr int kKVBytes = kChunk * D * 2;  // one of K or V for one chunk
  static constexpr int q = 0;
  static constexpr int k0 = q + kQBytes;
  static constexpr int v0 = k0 + kStages * kKVBytes;
  static constexpr int bars = v0 + kStages * kKVBytes;
  static constexpr int misc = bars + 24 * 8;
  static constexpr int bitmap = misc + 64;
  static constexpr int fixed = bitmap;  // + bitmap words
  // TMEM columns: S buffers [0,64) and [64,128) (P over the first 32 columns
  // of its own S buffer, bf16 pairs), O [128,128+D)
  static constexpr uint32_t kSCol = 0, kOCol = 128, kTmemCols = 256;
};

// K and V have their own barriers: a K slot frees when its QK^T is done, a V
// slot only when its PV is, so K can be fetched further ahead.  S buffer b:
// s_full (QK^T done), p_full (the rows stored P), p_free (PV read P).
struct Bars {
  uint64_t q, k_full[kStages], k_empty[kStages], v_full[kStages], v_empty[kStages], s_full[2],
      p_full[2], p_free[2], o_full, done, q_rot;
};
static_assert(sizeof(Bars) <= 24 * 8, "barrier area");

struct ChunkIter {
  const uint32_t *bm;
  int wi;
  uint32_t word;
  int n_own, own_next;  // own chunks: c0 + n_own - 1 down to c0
  __device__ void init(const uint32_t *b, int c0, int nown) {
    bm = b;
    wi = 0;
    word = b[0];
    n_own = nown;
    own_next = c0 + nown - 1;
  }
  __device__ int next() {
    if (n_own > 0) {
      --n_own;
      return own_next--;
    }
    while (word == 0) word = bm[++wi];
    const int c = wi * 32 + __ffs(word) - 1;
    word &= word - 1;
    return c;
  }
};

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

// acc_lo += low bf16 of w, acc_hi += high bf16 of w (each widened exactly
// to fp32, then one fp32 addition)
__device__ __forceinline__ void add_bf16x2_f32(float &acc_lo, float &acc_hi, uint32_t w) {
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "mov.b32 {lo, hi}, %2;\n\t"
      "add.rn.f32.bf16 %0, lo, %0;\n\t"
      "add.rn.f32.bf16 %1, hi, %1;\n\t}"
      : "+f"(acc_lo), "+f"(acc_hi)
      : "r"(w));
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// HoPE in place on row r of the swizzled bf16 Q tile (D/64 blocks of [128
// rows][128 bytes]) at position pos: element e pairs with e + D/2, i.e. the
// same 16-byte chunk of the other block (D = 128) or the chunk four chunks
// away in the same block (D = 64).
template <int D>
__device__ __forceinline__ void hope_row_inplace(unsigned char *tile, int r, const HopeParams &hp,
                                                 long long pos) {
  constexpr int HALF = D / 2;
#pragma unroll 1
  for (int j = 0; j < (D == 128 ? 8 : 4); ++j) {
    // first-half chunk (block 0, chunk j) and its partner
    unsigned char *pa = tile + r * 128 + ((j ^ (r & 7)) << 4);
    unsigned char *pb = D == 128 ? tile + kRows * 128 + r * 128 + ((j ^ (r & 7)) << 4)
                                 : tile + r * 128 + (((j + 4) ^ (r & 7)) << 4);
    uint4 a4 = *reinterpret_cast<const uint4 *>(pa);
    uint4 b4 = *reinterpret_cast<const uint4 *>(pb);
    uint32_t aw[4] = {a4.x, a4.y, a4.z, a4.w}, bw[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      float ya[2], yb[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int i = 8 * j + 2 * m + u;  // the pair (first element i < HALF)
        const float xi = __uint_as_float(u ? (aw[m] & 0xFFFF0000u) : (aw[m] << 16));
        const float xj = __uint_as_float(u ? (bw[m] & 0xFFFF0000u) : (bw[m] << 16));
        ya[u] = xi;
        yb[u] = xj;
        if (i < hp.npairs && i < HALF) {
          float sn, cs;
          hope_sincos(hp.turns[i], pos, sn, cs);
          hope_rotate(xi, xj, sn, cs, ya[u], yb[u]);
        }
      }
      const __nv_bfloat162 a2 = __floats2bfloat162_rn(ya[0], ya[1]);
      const __nv_bfloat162 b2 = __floats2bfloat162_rn(yb[0], yb[1]);
      aw[m] = *reinterpret_cast<const uint32_t *>(&a2);
      bw[m] = *reinterpret_cast<const uint32_t *>(&b2);
    }
    *reinterpret_cast<uint4 *>(pa) = make_uint4(aw[0], aw[1], aw[2], aw[3]);
    *reinterpret_cast<uint4 *>(pb) = make_uint4(bw[0], bw[1], bw[2], bw[3]);
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
    attn_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, RowSpec rs,
                      const int32_t *__restrict__ sel, const float *__restrict__ chunk_w,
                      __nv_bfloat16 *__restrict__ out, float *__restrict__ lse_out,
                      float *__restrict__ wfin, uint32_t *__restrict__ err,
                      const HopeParams hp) {
  using Lay = Layout<D>;
  // The 128-byte-swizzled tiles need a 1024-byte aligned base; the dynamic
  // shared window starts there (no static shared memory), checked here.
  extern __shared__ __align__(1024) unsigned char smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) report(err, DEV_BAD_INDEX);
    return;
  }
  Bars *bars = reinterpret_cast<Bars *>(smem + Lay::bars);
  uint32_t *tmem_base_slot = reinterpret_cast<uint32_t *>(smem + Lay::misc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Lay::misc + 4);
  int *n_steps_slot = reinterpret_cast<int *>(smem + Lay::misc + 8);
  uint32_t *bitmap = reinterpret_cast<uint32_t *>(smem + Lay::bitmap);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int b = bh / rs.Hq, hq = bh % rs.Hq, hkv = hq / (rs.Hq / rs.Hkv);
  const uint64_t lim = rs.wait_ns;
  const int t0 = blockIdx.x * kRows;
  const int L = rs.L, K = rs.topk;
  const int nchunks = (L + kChunk - 1) / kChunk;
  const int nwords = (nchunks + 31) / 32 + 1;  // +1: a zero guard word
  const int c0 = t0 / kChunk;
  const int n_own = (t0 + kChunk < L) ? 2 : 1;

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    mbar_init(&bars->q, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int b2 = 0; b2 < 2; ++b2) {
      mbar_init(&bars->s_full[b2], 1);
      mbar_init(&bars->p_full[b2], kRows);
      mbar_init(&bars->p_free[b2], 1);
    }
    mbar_init(&bars->o_full, 1);
    mbar_init(&bars->done, 1);
    mbar_init(&bars->q_rot, kRows);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_slot, Lay::kTmemCols);
    tmem_relinquish();
  }
  for (int i = threadIdx.x; i < nwords; i += kThreads) bitmap[i] = 0;
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_slot;

  // ------------------------------------------------ per-row prologue (warps 2-5)
  const bool is_row = warp >= 2;
  const int r = 32 * (warp & 3) + lane;  // TMEM lane == tile row
  const int t = t0 + r;
  const bool valid = is_row && t < L;
  const int own = t / kChunk;
  const size_t row = (size_t)bh * L + t;
  const int32_t *mysel = sel + row * K;
  const float *myw = chunk_w + row * K;
  int nsel = 0, walk_n = 0;
  float wmax2 = -INFINITY, sumsel = 0.0f, w_c0 = 0.0f;
  bool has_c0 = false;
  if (valid) {
    // the row's selection, 16 entries per round with all loads in flight
    // together: ids ascending with -1 padding at the end, and their logits;
    // a running maximum / rescaled sum gives sum_c exp(s_c - max) (base 2)
    int last_c = -1;
    float last_w2 = 0.0f;
    bool done = false;
    for (int i0 = 0; i0 < K && !done; i0 += 16) {
      int cc[16];
      float ww[16];
      if ((K & 3) == 0) {
#pragma unroll
        for (int u = 0; u < 16; u += 4) {
          const bool in = i0 + u < K;
          const int4 c4 = in ? __ldg(reinterpret_cast<const int4 *>(mysel + i0 + u)) : make_int4(-1, -1, -1, -1);
          const float4 w4 = in ? __ldg(reinterpret_cast<const float4 *>(myw + i0 + u)) : make_float4(0.f, 0.f, 0.f, 0.f);
          cc[u] = c4.x; cc[u + 1] = c4.y; cc[u + 2] = c4.z; cc[u + 3] = c4.w;
          ww[u] = w4.x; ww[u + 1] = w4.y; ww[u + 2] = w4.z; ww[u + 3] = w4.w;
        }
      } else {
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const bool in = i0 + u < K;
          cc[u] = in ? __ldg(mysel + i0 + u) : -1;
          ww[u] = in ? __ldg(myw + i0 + u) : 0.0f;
        }
      }
      float gm = -INFINITY;
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int c = cc[u];
        if (done || c < 0) {
          done = true;
          cc[u] = -1;
          continue;
        }
        if (c >= own) {
          report(err, DEV_BAD_INDEX);
          done = true;
          cc[u] = -1;
          continue;
        }
        atomicOr(&bitmap[c >> 5], 1u << (c & 31));
        ww[u] *= kLog2e;
        gm = fmaxf(gm, ww[u]);
        last_c = c;
        last_w2 = ww[u];
        ++nsel;
      }
      if (gm > wmax2) {
        sumsel *= ex2_approx(wmax2 - gm);
        wmax2 = gm;
      }
#pragma unroll
      for (int u = 0; u < 16; ++u)
        if (cc[u] >= 0) sumsel += ex2_approx(ww[u] - wmax2);
    }
    walk_n = nsel;
    if (own == c0 + 1 && nsel > 0 && last_c == c0) {
      has_c0 = true;
      w_c0 = last_w2;
      walk_n = nsel - 1;
    }
  }
  __syncthreads();
  if (warp == 0) {
    // own chunks are processed first; take them out of the ascending walk
    if (lane == 0) {
      bitmap[c0 >> 5] &= ~(1u << (c0 & 31));
      if (c0 + 1 < nchunks) bitmap[(c0 + 1) >> 5] &= ~(1u << ((c0 + 1) & 31));
    }
    __syncwarp();
    int cnt = 0;
    for (int i = lane; i < nwords; i += 32) cnt += __popc(bitmap[i]);
    for (int o = 16; o; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (lane == 0) *n_steps_slot = n_own + cnt;
  }
  __syncthreads();
  const int n_steps = *n_steps_slot;

  const uint32_t s_tmem = tmem + Lay::kSCol;  // buffer b at s_tmem + 64 b
  const uint32_t o_tmem = tmem + Lay::kOCol;
  unsigned char *q_s = smem + Lay::q;
  const int kv_row0 = (b * rs.Hkv + hkv) * L;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_expect_tx(&bars->q, Lay::kQBytes);
      for (int kb = 0; kb < D / 64; ++kb)
        tma_load_2d(q_s + kb * kRows * 128, &tm_q, &bars->q, kb * 64, bh * L + t0);
      // K runs one step ahead of V in the issue order: K(j + 1) waits only
      // for QK^T(j - 1), V(j) for PV(j - 2)
      ChunkIter itk, itv;
      itk.init(bitmap, c0, n_own);
      itv.init(bitmap, c0, n_own);
      int k_issued = 0, v_issued = 0;
      auto load_k = [&](int j) -> bool {
        const int c = itk.next();
        const int s = j % kStages;
        if (j >= kStages && !mbar_wait(&bars->k_empty[s], ((j / kStages) - 1) & 1, abort_flag, lim))
          return false;
        mbar_expect_tx(&bars->k_full[s], Lay::kKVBytes);
        unsigned char *ks = smem + Lay::k0 + s * Lay::kKVBytes;
        for (int kb = 0; kb < D / 64; ++kb)
          tma_load_2d(ks + kb * kChunk * 128, &tm_k, &bars->k_full[s], kb * 64, kv_row0 + c * kChunk);
        ++k_issued;
        return true;
      };
      auto load_v = [&](int j) -> bool {
        const int c = itv.next();
        const int s = j % kStages;
        if (j >= kStages && !mbar_wait(&bars->v_empty[s], ((j / kStages) - 1) & 1, abort_flag, lim))
          return false;
        mbar_expect_tx(&bars->v_full[s], Lay::kKVBytes);
        unsigned char *vs = smem + Lay::v0 + s * Lay::kKVBytes;
        for (int kb = 0; kb < D / 64; ++kb)
          tma_load_2d(vs + kb * kChunk * 128, &tm_v, &bars->v_full[s], kb * 64, kv_row0 + c * kChunk);
        ++v_issued;
        return true;
      };
      bool ok = n_steps > 0 ? load_k(0) : true;
      for (int j = 0; ok && j < n_steps; ++j) {
        if (j + 1 < n_steps) ok = load_k(j + 1);
        if (ok) ok = load_v(j);
      }
      // every load issued must land before the CTA may exit
      for (int i = (k_issued > kStages ? k_issued - kStages : 0); i < k_issued; ++i)
        mbar_wait_bounded(&bars->k_full[i % kStages], (i / kStages) & 1, lim);
      for (int i = (v_issued > kStages ? v_issued - kStages : 0); i < v_issued; ++i)
        mbar_wait_bounded(&bars->v_full[i % kStages], (i / kStages) & 1, lim);
      mbar_wait_bounded(&bars->q, 0, lim);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kRows, kChunk, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kRows, D, false, true);
      const uint32_t q_addr = smem_u32(q_s);
      // S_j = Q K_j^T into S buffer j & 1, once K_j has landed and PV_{j-2}
      // has read P_{j-2} from that buffer
      auto qk = [&](int j) -> bool {
        const int s = j % kStages, b2 = j & 1;
        if (!mbar_wait(&bars->k_full[s], (j / kStages) & 1, abort_flag, lim)) return false;
        if (j >= 2 && !mbar_wait(&bars->p_free[b2], ((j >> 1) - 1) & 1, abort_flag, lim)) return false;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(smem + Lay::k0 + s * Lay::kKVBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int kb = kk >> 2, kw = kk & 3;
          const uint64_t a = smem_desc_sw128(q_addr + kb * kRows * 128 + kw * 32, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(k_addr + kb * kChunk * 128 + kw * 32, 16, 1024);
          mma_bf16_ss(s_tmem + 64 * b2, a, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars->s_full[b2]);
        mma_commit(&bars->k_empty[s]);
        return true;
      };
      // O += P_j V_j, P_j read from the first 32 columns of S buffer j & 1
      auto pv = [&](int j) -> bool {
        const int s = j % kStages, b2 = j & 1;
        if (!mbar_wait(&bars->v_full[s], (j / kStages) & 1, abort_flag, lim)) return false;
        if (!mbar_wait(&bars->p_full[b2], (j >> 1) & 1, abort_flag, lim)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(smem + Lay::v0 + s * Lay::kKVBytes);
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk) {
          // A = P [128 x 64] in tensor memory: 16 keys = 8 columns
          // B = V [64 keys x D] MN-major: 16 keys = 16 rows of 128 bytes;
          // the D axis is split into 64-wide blocks 64*128 bytes apart
          const uint64_t bdesc = smem_desc_sw128(v_addr + kk * 16 * 128, kChunk * 128, 1024);
          mma_bf16_ts(o_tmem, s_tmem + 64 * b2 + kk * 8, bdesc, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&bars->v_empty[s]);
        mma_commit(&bars->p_free[b2]);
        return true;
      };
      // with HoPE the rows turn the Q tile before the first QK^T reads it
      bool ok = hp.npairs > 0 ? mbar_wait(&bars->q_rot, 0, abort_flag, lim)
                              : mbar_wait(&bars->q, 0, abort_flag, lim);
      if (ok) ok = qk(0);
      if (ok && n_steps > 1) ok = qk(1);
      for (int j = 0; ok && j < n_steps; ++j) {
        ok = pv(j);
        if (ok && j + 2 < n_steps) ok = qk(j + 2);
      }
      if (ok) mma_commit(&bars->o_full);
      // all issued tensor-core work must finish before TMEM is released
      mma_commit(&bars->done);
      mbar_wait_bounded(&bars->done, 0, lim);
    }
  } else {
    // ------------------------------------------------------------ softmax rows
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const float scale2 = rs.scale * kLog2e;
    float M2 = 0.0f, lse2_own = 0.0f;
    int ptr = 0;
    bool ok = true;
    // the row's next four selected chunks (ids and logits), loaded ahead so
    // that a global load has several steps to land before it is used
    int qc[4];
    float qw[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const bool have = valid && u < walk_n;
      qc[u] = have ? __ldg(mysel + u) : -1;
      qw[u] = have ? __ldg(myw + u) : 0.0f;
    }
    if (hp.npairs > 0) {
      // HoPE on the fly: each row turns its own line of the Q tile once the
      // tile has landed; the generic-proxy writes are fenced for the tensor
      // core before the arrival the MMA issuer waits on
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->q, 0, abort_flag, lim));
      if (ok) hope_row_inplace<D>(q_s, r, hp, (long long)hp.pos0 + t);
      fence_async_smem();
      mbar_arrive(&bars->q_rot);
    }
    ChunkIter it;
    it.init(bitmap, c0, n_own);
    // sum of the rounded probabilities this row stores (four partial sums)
    float rsum[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    for (int i = 0; ok && i < n_steps; ++i) {
      const int c = it.next();
      const uint32_t sb = s_tmem + 64 * (i & 1) + lane_off;
      ok = mbar_wait(&bars->s_full[i & 1], (i >> 1) & 1, abort_flag, lim);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      float x[64];
      {
        float (&x0)[32] = *reinterpret_cast<float (*)[32]>(&x[0]);
        float (&x1)[32] = *reinterpret_cast<float (*)[32]>(&x[32]);
        tmem_ld32(sb, x0);
        tmem_ld32(sb + 32, x1);
        tmem_wait_ld();
      }

      // does this row attend chunk c, and with which logit?
      int kind = 0;  // 0 none, 1 own, 2 selected
      float logit2 = 0.0f;
      if (valid) {
        if (c == own) {
          kind = 1;
        } else if (c == c0 && has_c0) {
          kind = 2;
          logit2 = w_c0;
        } else if (ptr < walk_n && c == qc[0]) {
          kind = 2;
          logit2 = qw[0] * kLog2e;
          ++ptr;
          qc[0] = qc[1];
          qc[1] = qc[2];
          qc[2] = qc[3];
          qw[0] = qw[1];
          qw[1] = qw[2];
          qw[2] = qw[3];
          const bool have = ptr + 3 < walk_n;
          qc[3] = have ? __ldg(mysel + ptr + 3) : -1;
          qw[3] = have ? __ldg(myw + ptr + 3) : 0.0f;
        }
      }
      // Rows of the warp that do not attend chunk c run the same softmax on
      // their (finite) scores and scale it by 0, so the warp takes one path.
      uint32_t pk[32];
      if (__any_sync(0xffffffffu, kind != 0)) {
        if (kind == 1) {  // causal keys of the own chunk
          const int jmax = t - c * kChunk;
#pragma unroll
          for (int j = 0; j < 64; ++j) x[j] = (j <= jmax) ? x[j] : -INFINITY;
        }
        float mx[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) mx[j] = fmaxf(fmaxf(x[j], x[j + 16]), fmaxf(x[j + 32], x[j + 48]));
#pragma unroll
        for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
          for (int j = 0; j < w; ++j) mx[j] = fmaxf(mx[j], mx[j + w]);
        const float m2 = mx[0] * scale2;
        // elementwise fp32 work on pairs (packed f32x2 FMA / add / multiply)
        const float2 c2v = make_float2(scale2, scale2), nm2 = make_float2(-m2, -m2);
        float2 ls[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float2 y = __ffma2_rn(make_float2(x[2 * j], x[2 * j + 1]), c2v, nm2);
          x[2 * j] = ex2_approx(y.x);
          x[2 * j + 1] = ex2_approx(y.y);
          ls[j & 1] = __fadd2_rn(ls[j & 1], make_float2(x[2 * j], x[2 * j + 1]));
        }
        const float l = (ls[0].x + ls[1].x) + (ls[0].y + ls[1].y);
        float sc;
        if (kind == 1) {
          lse2_own = m2 + __log2f(l);
          M2 = fmaxf(lse2_own, wmax2);
          sc = ex2_approx(m2 - M2);
        } else if (kind == 2) {
          sc = __fdividef(ex2_approx(logit2 - M2), l);  // l in [1, 64]
        } else {
          sc = 0.0f;
        }
        const float2 scv = make_float2(sc, sc);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float2 pj = __fmul2_rn(make_float2(x[2 * j], x[2 * j + 1]), scv);
          pk[j] = pack_bf16(pj.x, pj.y);
          add_bf16x2_f32(rsum[2 * (j & 1)], rsum[2 * (j & 1) + 1], pk[j]);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) pk[j] = 0u;
      }
      // P over the S just read (this buffer is the rows' until p_full)
      __syncwarp();  // tcgen05.st is warp-collective
      tmem_st32(sb, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->p_full[i & 1]);
    }
    // ---------------------------------------------------------- epilogue
    if (ok) ok = mbar_wait(&bars->o_full, 0, abort_flag, lim);
    if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after();
      const float lsum = ex2_approx(lse2_own - M2) + sumsel * ex2_approx(wmax2 - M2);
      const float lsum_rounded = (rsum[0] + rsum[2]) + (rsum[1] + rsum[3]);
      const float inv = 1.0f / lsum_rounded;
      __nv_bfloat16 *orow = out + row * D;
#pragma unroll
      for (int cb = 0; cb < D / 32; ++cb) {
        float o[32];
        tmem_ld32(o_tmem + lane_off + cb * 32, o);
        tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint4 v4 = make_uint4(pack_bf16(o[8 * j] * inv, o[8 * j + 1] * inv),
                                  pack_bf16(o[8 * j + 2] * inv, o[8 * j + 3] * inv),
                                  pack_bf16(o[8 * j + 4] * inv, o[8 * j + 5] * inv),
                                  pack_bf16(o[8 * j + 6] * inv, o[8 * j + 7] * inv));
            *reinterpret_cast<uint4 *>(orow + cb * 32 + 8 * j) = v4;
          }
        }
      }
      if (valid) {
        const float lse2 = M2 + __log2f(lsum);
        lse_out[row] = lse2 * kLn2;
        if (wfin) {
          float *wr = wfin + row * (K + 1);
          for (int i = 0; i < K; ++i)
            wr[i] = i < nsel ? exp2f(__ldg(myw + i) * kLog2e - lse2) : 0.0f;
          wr[K] = exp2f(lse2_own - lse2);
        }
        if (ptr != walk_n) report(err, DEV_BAD_INDEX);
      }
    }
  }
  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) report(err, DEV_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Lay::kTmemCols);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// 2-D tensor map over a row-major [rows, cols] array of 2- or 4-byte
// elements with a [box_rows, 128 bytes] box and 128-byte swizzle.
static cudaError_t make_tmap_2d(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                                uint32_t box_rows, bool f32) {
  static EncodeTiledFn encode = nullptr;
  if (!encode) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
    encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  const uint32_t esz = f32 ? 4 : 2;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * esz};
  const cuuint32_t box[2] = {128 / esz, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                      2, const_cast<void *>(base), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

cudaError_t make_tmap_bf16(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                           uint32_t box_rows) {
  return make_tmap_2d(map, base, rows, cols, box_rows, false);
}

cudaError_t make_tmap_f32(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                          uint32_t box_rows) {
  return make_tmap_2d(map, base, rows, cols, box_rows, true);
}

size_t attn_sm100_smem(int d, int L) {
  const int nwords = ((L + 63) / 64 + 31) / 32 + 1;
  const size_t fixed = d == 64 ? Layout<64>::fixed : Layout<128>::fixed;
  return fixed + (size_t)nwords * 4;
}

cudaError_t attn_sm100(const RowSpec &rs, const void *q, const void *k, const void *v,
                       const int32_t *sel, const float *w, void *out, float *lse, float *wfin,
                       uint32_t *err, cudaStream_t st, const HopeParams &hp) {
  CUtensorMap tq, tk, tv;
  cudaError_t e;
  const uint64_t qrows = (uint64_t)rs.B * rs.Hq * rs.L, kvrows = (uint64_t)rs.B * rs.Hkv * rs.L;
  if ((e = make_tmap_bf16(&tq, q, qrows, rs.d, kRows)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&tk, k, kvrows, rs.d, kChunk)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&tv, v, kvrows, rs.d, kChunk)) != cudaSuccess) return e;
  const size_t smem = attn_sm100_smem(rs.d, rs.L);
  dim3 grid((rs.L + kRows - 1) / kRows, rs.B * rs.Hq);
  if (rs.d == 64) {
    auto kern = attn_sm100_kernel<64>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess) return e;
    kern<<<grid, kThreads, smem, st>>>(tq, tk, tv, rs, sel, w, (__nv_bfloat16 *)out, lse, wfin, err, hp);
  } else {
    auto kern = attn_sm100_kernel<128>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess) return e;
    kern<<<grid, kThreads, smem, st>>>(tq, tk, tv, rs, sel, w, (__nv_bfloat16 *)out, lse, wfin, err, hp);
  }
  return cudaGetLastError();
}

}  // namespace hils
