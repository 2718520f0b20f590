// Landmark scoring, inter-chunk normaliser and top-k chunk selection on the
// 5th-generation tensor cores (model card "HiLS-Attention", section "What
// HiLS-Attention is"; molayo1419.me, "Core idea" step 1): for every query row
// t the logits s_c = scale * <q_t, lmk_c> of its completed chunks c < t/C,
// their log-sum-exp, and the k best by (s desc, c asc).
//
// One CTA = 128 query rows of one (b, hq); two CTAs share an SM.  10 warps:
//   warp 0     TMA producer: the Q tile into the landmark ring (staging), then
//              64-landmark tiles of the row block's KV head into a 2-stage
//              ring, each with a small bias tile (below) written beside it;
//   warp 1     TMEM owner, MMA issuer: the seed scores, then per landmark tile
//              S = Q Lmk^T + bias (128 x 64 fp32) into one of two TMEM
//              buffers, with Q as the A operand in tensor memory;
//   warps 2-9  two threads per row: warps 2-5 (the row's "owner") read columns
//              [0, 32) of every score tile, warps 6-9 columns [32, 64).  Each
//              keeps an online log-sum-exp (base 2) of its half; the row's
//              best k keys live in shared memory and only the owner changes
//              them: the other thread posts the candidates that beat the
//              row's threshold into a 4-entry mailbox the owner drains once
//              per tile.
// Seeds.  Every row's top-k starts from k chunks (the seeds) whose scores an
// extra MMA computes first: the k-th best seed bounds the row's k-th best
// score from below (the seeds are candidates too), so the result stays exact
// and the scan only inserts what beats that bound.  The row tiles run in
// kLevels launches: tiles of level 0 start from the chunks 0..k-1 (where a
// plain scan starts), tiles of later levels from the selection of the last
// row of a tile an earlier level finished (1, 2, 4, ... tiles before them),
// which adjacent queries largely share.
// Masking on the tensor core.  The seeds (already counted, in the top-k and
// in the log-sum-exp, from their own MMA) and the chunks a row may not see
// (the tile's first own chunk for its first 64 rows, and every column past
// the tile's last candidate) are pushed to -1e30 by one more K = 16 step of
// the scoring MMA: A = [1, (row < 64)] per row (8 TMEM columns), B = per
// landmark column [-1e30 if a seed or beyond the candidates, -1e30 if the
// boundary chunk] (written by the producer while the tile's TMA is in
// flight, and only for tiles that hold a seed or the boundary).  For every
// other column that step adds exact zeros, so the scores are unchanged; the
// row threads then need no per-block masks, and blocks holding seeds no
// longer pass the top-k prefilter.
// The candidate scores never leave the chip.
#include <cuda_bf16.h>

#include "common.cuh"
#include "hope.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace hils {
namespace {

using namespace sm100;

constexpr int kRows = 128;
constexpr int kTile = 64;     // landmarks per MMA tile (UMMA N)
constexpr int kStages = 2;    // landmark ring
constexpr int kSBufs = 2;     // score tiles in tensor memory
constexpr int kRowThreads = 2 * kRows;
constexpr int kThreads = 64 + kRowThreads;
constexpr int kMaxK = 64;
constexpr int kMbox = 4;      // mailbox entries per row
constexpr uint32_t kDone = 0x80000000u;
// a score below this (unscaled) was pushed down by the masking step
constexpr float kMaskedBelow = -1.0e29f;
// Row tiles run in kLevels launches (levels): with P = 2^(kLevels-1), level 0
// takes the tiles P*i unseeded and level j >= 1 the tiles at offset P/2^j in
// periods of P/2^(j-1), each seeded by the tile offset positions earlier
// (which an earlier level finished).
#ifndef HILS_SELECT_LEVELS
#define HILS_SELECT_LEVELS 6
#endif
constexpr int kLevels = HILS_SELECT_LEVELS;
constexpr int kLevelP = 1 << (kLevels - 1);
__host__ __device__ constexpr int level_period(int lv) { return lv == 0 ? kLevelP : (kLevelP >> (lv - 1)); }
__host__ __device__ constexpr int level_offset(int lv) { return lv == 0 ? 0 : (kLevelP >> lv); }
__host__ __device__ inline int level_count(int lv, int ntiles) {
  const int p = level_period(lv), o = level_offset(lv);
  return ntiles > o ? (ntiles - o + p - 1) / p : 0;
}
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <int D>
struct SelLayout {
  static constexpr int kQBytes = kRows * D * 2;
  static constexpr int kLBytes = kTile * D * 2;
  static_assert(kStages * kLBytes == kQBytes, "the landmark ring stages the Q tile");
  static constexpr int l0 = 0;                               // landmark ring / Q / seed staging
  static constexpr int bias = l0 + kStages * kLBytes;        // [64 rows][128 B], 128-byte swizzle
  static constexpr int heap = bias + kTile * 128;            // [kMaxK][128] uint64 slots
  static constexpr int mbox = heap + kMaxK * kRows * 8;      // [kMbox][128] uint64 keys
  static constexpr int tail = mbox + kMbox * kRows * 8;      // [128] posted count (+ done bit)
  static constexpr int head = tail + kRows * 4;              // [128] drained count
  static constexpr int thr = head + kRows * 4;               // [128] prefilter bound
  static constexpr int lsep = thr + kRows * 4;               // [128] (m2, l) of the second half
  static constexpr int bars = lsep + kRows * 8;
  static constexpr int misc = bars + 16 * 8;
  static constexpr int seeds = misc + 32;                     // [kMaxK] int seed chunk ids
  static constexpr int total = seeds + kMaxK * 4;
  static_assert(bias % 1024 == 0, "swizzled tiles are 1024-byte aligned");
  // the epilogue's per-warp staging blocks [32][64 + 4] words (4 owner warps)
  // in the landmark ring and the masking tile that follows it, where they fit
  // (d = 128; at d = 64 the rows are written directly)
  static constexpr bool kStagedOut = 4 * 32 * (kMaxK + 4) * 4 <= heap - l0;
  // TMEM columns: Q [0, D/2) as bf16 pairs, the masking A operand [64, 72),
  // score buffers [128, 192) and [192, 256)
  static constexpr uint32_t kQCol = 0, kBiasCol = 64, kSCol = 128, kTmemCols = 256;
  static_assert(kSCol + kSBufs * kTile <= kTmemCols, "score tiles fit the allocation");
};

struct SelBars {
  uint64_t q_smem, q_tmem, l_full[kStages], l_empty[kStages], s_full[kSBufs], s_empty[kSBufs],
      seed_ready, seed_full, seed_read, seed_done, done;
};
static_assert(sizeof(SelBars) <= 16 * 8, "barrier area");

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
  float thr;      // score of mn

  __device__ __forceinline__ void rescan(const uint64_t *h, int g, int K) {
    uint64_t x[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int slot = g * 8 + i;
      x[i] = slot < K ? h[slot * kRows] : ~0ull;
    }
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
    gpos = 0;
#pragma unroll 1
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

// Prefilter bound in the unscaled domain: every a with fl(a * scale) >= thr
// satisfies a >= prefilter(thr, 1 / scale).  The product and thr * (1/scale)
// each round by at most 2^-24 relative; the bound leaves 2^-20 plus an
// absolute 2^-100.  Candidates that pass are decided exactly on their key.
__device__ __forceinline__ float prefilter(float thr, float inv_scale) {
  if (isinf(thr)) return thr;
  const float u = thr * inv_scale;
  return u - fabsf(u) * 0x1p-20f - 0x1p-100f;
}

// a[j] for a j known only at run time, by a tree of selects (no local memory)
__device__ __forceinline__ float pick32(const float (&a)[32], int j) {
  float b16[16], b8[8], b4[4], b2[2];
#pragma unroll
  for (int i = 0; i < 16; ++i) b16[i] = (j & 16) ? a[i + 16] : a[i];
#pragma unroll
  for (int i = 0; i < 8; ++i) b8[i] = (j & 8) ? b16[i + 8] : b16[i];
#pragma unroll
  for (int i = 0; i < 4; ++i) b4[i] = (j & 4) ? b8[i + 4] : b8[i];
#pragma unroll
  for (int i = 0; i < 2; ++i) b2[i] = (j & 2) ? b4[i + 2] : b4[i];
  return (j & 1) ? b2[1] : b2[0];
}

// Writes a row's first cnt kept keys in slot order (ids, logits; -1 / -inf
// padding up to K).
__device__ __forceinline__ void write_in_order(const uint64_t *slots, int cnt, int K,
                                               int32_t *__restrict__ srow,
                                               float *__restrict__ wrow) {
  if ((K & 3) == 0) {
#pragma unroll 1
    for (int i = 0; i < K; i += 4) {
      int4 si;
      float4 wi;
      int *sp4 = &si.x;
      float *wp4 = &wi.x;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const bool have = i + u < cnt;
        const uint64_t x = have ? slots[(i + u) * kRows] : 0;
        sp4[u] = have ? key_chunk(x) : -1;
        wp4[u] = have ? key_score(x) : -INFINITY;
      }
      *reinterpret_cast<int4 *>(srow + i) = si;
      *reinterpret_cast<float4 *>(wrow + i) = wi;
    }
  } else {
#pragma unroll 1
    for (int i = 0; i < K; ++i) {
      const bool have = i < cnt;
      const uint64_t x = have ? slots[i * kRows] : 0;
      srow[i] = have ? key_chunk(x) : -1;
      wrow[i] = have ? key_score(x) : -INFINITY;
    }
  }
}

// Sorts a full row's K kept keys by chunk id and writes them.  Chunk ids are
// below 2^25 (L < 2^31, C = 64), so (id << 6 | slot) fits a 32-bit word; a
// bitonic network of N/2 log N (log N + 1) / 2 min/max pairs sorts N words in
// registers without branches (words past K sort last).
// The warp's 32 rows (K = N = 32 or 64, every row searched) written through
// a per-warp staging block [32][N + 4] words in shared memory: each lane
// sorts its row's (chunk << 6 | slot) words as write_sorted does and stores
// them as a row of the block (a row stride of 4 mod 32 words keeps the
// 16-byte accesses free of bank conflicts); the warp copies the chunk ids out
// with coalesced 16-byte stores (two 256-byte rows per instruction for
// N = 64); each lane then replaces its row's words by their logits, read from
// its slots, and the warp copies those out the same way.  rows_valid: the
// warp's rows below L.
template <int N, bool kIds>
__device__ __forceinline__ void copy_block_out(const uint32_t *stage, int lane,
                                               uint32_t *__restrict__ dst, int rows_valid) {
  constexpr int S = N + 4, P = N / 4;  // staging stride (words), 16-byte pieces per row
#pragma unroll
  for (int u = 0; u < P; ++u) {
    const int pc = u * 32 + lane, row = pc / P, c = pc % P;
    if (row < rows_valid) {
      uint4 x = *reinterpret_cast<const uint4 *>(stage + row * S + 4 * c);
      if (kIds) x = make_uint4(x.x >> 6, x.y >> 6, x.z >> 6, x.w >> 6);
      *reinterpret_cast<uint4 *>(dst + (size_t)row * N + 4 * c) = x;
    }
  }
}

template <int N>
__device__ __forceinline__ void write_sorted_staged(const uint64_t *slots, uint32_t *stage,
                                                    int lane, int32_t *__restrict__ sel_w,
                                                    float *__restrict__ w_w, int rows_valid) {
  constexpr int S = N + 4;
  uint32_t *mine = stage + lane * S;
  {
    uint32_t v[N];
#pragma unroll
    for (int i = 0; i < N; ++i) {
      const uint32_t lo = reinterpret_cast<const uint32_t *>(slots + i * kRows)[0];
      v[i] = ((0xFFFFFFFFu - lo) << 6) | (uint32_t)i;
    }
#pragma unroll
    for (int size = 2; size <= N; size <<= 1)
#pragma unroll
      for (int stride = size >> 1; stride > 0; stride >>= 1)
#pragma unroll
        for (int i = 0; i < N; ++i) {
          const int j = i ^ stride;
          if (j > i) {
            const uint32_t x = v[i], y = v[j];
            const bool up = (i & size) == 0;
            v[i] = up ? min(x, y) : max(x, y);
            v[j] = up ? max(x, y) : min(x, y);
          }
        }
#pragma unroll
    for (int i = 0; i < N; i += 4)
      *reinterpret_cast<uint4 *>(mine + i) = make_uint4(v[i], v[i + 1], v[i + 2], v[i + 3]);
  }
  __syncwarp();
  copy_block_out<N, true>(stage, lane, reinterpret_cast<uint32_t *>(sel_w), rows_valid);
  __syncwarp();
#pragma unroll 4
  for (int i = 0; i < N; i += 4) {
    const uint4 x = *reinterpret_cast<const uint4 *>(mine + i);
    *reinterpret_cast<uint4 *>(mine + i) =
        make_uint4(__float_as_uint(key_score(slots[(x.x & 63u) * kRows])),
                   __float_as_uint(key_score(slots[(x.y & 63u) * kRows])),
                   __float_as_uint(key_score(slots[(x.z & 63u) * kRows])),
                   __float_as_uint(key_score(slots[(x.w & 63u) * kRows])));
  }
  __syncwarp();
  copy_block_out<N, false>(stage, lane, reinterpret_cast<uint32_t *>(w_w), rows_valid);
}

template <int N>
__device__ __forceinline__ void write_sorted(const uint64_t *slots, int K,
                                             int32_t *__restrict__ srow,
                                             float *__restrict__ wrow) {
  uint32_t v[N];
#pragma unroll
  for (int i = 0; i < N; ++i) {
    const uint32_t lo = i < K ? reinterpret_cast<const uint32_t *>(slots + i * kRows)[0] : 0u;
    v[i] = i < K ? (((0xFFFFFFFFu - lo) << 6) | (uint32_t)i) : 0xFFFFFFFFu;
  }
#pragma unroll
  for (int size = 2; size <= N; size <<= 1)
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1)
#pragma unroll
      for (int i = 0; i < N; ++i) {
        const int j = i ^ stride;
        if (j > i) {
          const uint32_t x = v[i], y = v[j];
          const bool up = (i & size) == 0;
          v[i] = up ? min(x, y) : max(x, y);
          v[j] = up ? max(x, y) : min(x, y);
        }
      }
  if ((K & 3) == 0) {
#pragma unroll
    for (int i = 0; i < N; i += 4) {
      if (i < K) {
        int4 si;
        float4 wi;
        si.x = (int)(v[i] >> 6);
        si.y = (int)(v[i + 1] >> 6);
        si.z = (int)(v[i + 2] >> 6);
        si.w = (int)(v[i + 3] >> 6);
        wi.x = key_score(slots[(v[i] & 63u) * kRows]);
        wi.y = key_score(slots[(v[i + 1] & 63u) * kRows]);
        wi.z = key_score(slots[(v[i + 2] & 63u) * kRows]);
        wi.w = key_score(slots[(v[i + 3] & 63u) * kRows]);
        *reinterpret_cast<int4 *>(srow + i) = si;
        *reinterpret_cast<float4 *>(wrow + i) = wi;
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < N; ++i) {
      if (i < K) {
        srow[i] = (int)(v[i] >> 6);
        wrow[i] = key_score(slots[(v[i] & 63u) * kRows]);
      }
    }
  }
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// The two threads of every row (warps 2-9) meet here.
__device__ __forceinline__ void rows_sync() {
  __syncwarp();
  asm volatile("bar.sync 1, %0;" ::"n"(kRowThreads) : "memory");
}

__device__ __forceinline__ uint32_t ld_vol(const uint32_t *p) { return *reinterpret_cast<const volatile uint32_t *>(p); }
__device__ __forceinline__ void st_vol(uint32_t *p, uint32_t v) { *reinterpret_cast<volatile uint32_t *>(p) = v; }
__device__ __forceinline__ float ld_volf(const float *p) { return *reinterpret_cast<const volatile float *>(p); }
__device__ __forceinline__ void st_volf(float *p, float v) { *reinterpret_cast<volatile float *>(p) = v; }

// Online log-sum-exp (base 2) of one 32-candidate block with block maximum
// bm (unscaled); c2 = scale * log2(e).  Blocks whose every entry was masked
// (bm below kMaskedBelow) add nothing.
__device__ __forceinline__ void lse_block(const float (&a)[32], float bm, float c2, float &m2,
                                          float &l) {
  if (!(bm > kMaskedBelow)) return;
  const float bm2 = bm * c2;
  if (bm2 > m2) {
    l *= ex2_approx(m2 - bm2);
    m2 = bm2;
  }
  // pairs of candidates through packed f32x2 FMA and add
  const float2 c2v = make_float2(c2, c2), nm2 = make_float2(-m2, -m2);
  float2 ps[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float2 y = __ffma2_rn(make_float2(a[2 * j], a[2 * j + 1]), c2v, nm2);
    ps[j & 1] = __fadd2_rn(ps[j & 1], make_float2(ex2_approx(y.x), ex2_approx(y.y)));
  }
  l += (ps[0].x + ps[1].x) + (ps[0].y + ps[1].y);
}

__device__ __forceinline__ float block_max(const float (&a)[32]) {
  // a tree of three-input maxima (32 -> 11 -> 4 -> 1)
  float y[11];
#pragma unroll
  for (int j = 0; j < 10; ++j) y[j] = max3f(a[3 * j], a[3 * j + 1], a[3 * j + 2]);
  y[10] = fmaxf(a[30], a[31]);
  return max3f(max3f(y[0], y[1], y[2]), max3f(y[3], y[4], y[5]),
               max3f(y[6], y[7], max3f(y[8], y[9], y[10])));
}

// bit j set where a[j] >= u
__device__ __forceinline__ uint32_t ge_mask(const float (&a)[32], float u) {
  uint32_t mq[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int j = 0; j < 32; ++j) mq[j >> 3] |= a[j] >= u ? (1u << j) : 0u;
  return (mq[0] | mq[1]) | (mq[2] | mq[3]);
}

// Row r of a swizzled bf16 Q tile (D/64 blocks of [128 rows][128 bytes])
// with HoPE applied at position pos, into the row's tensor-memory columns
// from taddr on (two bf16 per column, as the tile packs them).  Pair i joins
// elements i and i + D/2; 16-byte chunk j of the first half (pairs 8j ..
// 8j+7) has its partners in chunk j of block 1 (D = 128) or chunk j + 4 of
// block 0 (D = 64).  The row's two threads split the chunks, h taking j = h,
// h+2, ..., so each angle is formed once per row; every chunk pair goes out
// as two 4-column stores (no register array is indexed by the rolled loop).
template <int D>
__device__ __forceinline__ void hope_row_split(const unsigned char *tile, int r, int h,
                                               const HopeParams &hp, long long pos,
                                               uint32_t taddr) {
  constexpr int kChunks = D / 16;  // 16-byte chunks in the first half
#pragma unroll 1
  for (int j = h; j < kChunks; j += 2) {
    const unsigned char *row = tile + r * 128;
    const uint4 a4 = *reinterpret_cast<const uint4 *>(row + ((j ^ (r & 7)) << 4));
    const uint4 b4 = D == 128
        ? *reinterpret_cast<const uint4 *>(row + kRows * 128 + ((j ^ (r & 7)) << 4))
        : *reinterpret_cast<const uint4 *>(row + (((j + 4) ^ (r & 7)) << 4));
    uint32_t aw[4] = {a4.x, a4.y, a4.z, a4.w}, bw[4] = {b4.x, b4.y, b4.z, b4.w};
    if (8 * j < hp.npairs) {
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        float ya[2], yb[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int i = 8 * j + 2 * m + u;
          ya[u] = __uint_as_float(u ? (aw[m] & 0xFFFF0000u) : (aw[m] << 16));
          yb[u] = __uint_as_float(u ? (bw[m] & 0xFFFF0000u) : (bw[m] << 16));
          if (i < hp.npairs) {
            float sn, cs;
            hope_sincos(hp.turns[i], pos, sn, cs);
            hope_rotate(ya[u], yb[u], sn, cs, ya[u], yb[u]);
          }
        }
        const __nv_bfloat162 a2 = __floats2bfloat162_rn(ya[0], ya[1]);
        const __nv_bfloat162 b2 = __floats2bfloat162_rn(yb[0], yb[1]);
        aw[m] = *reinterpret_cast<const uint32_t *>(&a2);
        bw[m] = *reinterpret_cast<const uint32_t *>(&b2);
      }
    }
    tmem_st4(taddr + 4 * j, aw);
    tmem_st4(taddr + D / 4 + 4 * j, bw);
  }
}

// One row's selection in ascending chunk order (rows that kept every
// candidate are already in order).
__device__ __forceinline__ void write_row(const uint64_t *slots, int n_c, int cnt, int K,
                                          int32_t *__restrict__ srow, float *__restrict__ wrow) {
  if (n_c <= K)
    write_in_order(slots, cnt, K, srow, wrow);
  else if (K <= 16)
    write_sorted<16>(slots, K, srow, wrow);
  else if (K <= 32)
    write_sorted<32>(slots, K, srow, wrow);
  else
    write_sorted<64>(slots, K, srow, wrow);
}

// The row's log-sum-exp from its two halves' (max, sum) in base 2.
__device__ __forceinline__ float row_lse(float2 o, float m2, float l, int n_c) {
  const float mm = fmaxf(m2, o.x);
  const float ls = (m2 > -INFINITY ? l * ex2_approx(m2 - mm) : 0.0f) +
                   (o.x > -INFINITY ? o.y * ex2_approx(o.x - mm) : 0.0f);
  return n_c > 0 ? (mm + __log2f(ls)) * kLn2 : -INFINITY;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
    select_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_l, RowSpec rs,
                        int32_t *__restrict__ sel, float *__restrict__ chunk_w,
                        float *__restrict__ lse_lmk, uint32_t *__restrict__ err, int level,
                        const __nv_bfloat16 *__restrict__ lmk_raw, const HopeParams hp) {
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
  volatile int *nseed_slot = reinterpret_cast<volatile int *>(smem + Lay::misc + 8);
  volatile int *bias_flag = reinterpret_cast<volatile int *>(smem + Lay::misc + 16);  // [kStages]
  int *seed_list = reinterpret_cast<int *>(smem + Lay::seeds);
  uint32_t *tail_s = reinterpret_cast<uint32_t *>(smem + Lay::tail);
  uint32_t *head_s = reinterpret_cast<uint32_t *>(smem + Lay::head);
  float *thr_s = reinterpret_cast<float *>(smem + Lay::thr);
  float2 *lsep_s = reinterpret_cast<float2 *>(smem + Lay::lsep);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int b = bh / rs.Hq, hq = bh % rs.Hq, hkv = hq / (rs.Hq / rs.Hkv);
  const uint64_t lim = rs.wait_ns;
  // this launch's level: tiles offset + i * period, heaviest first
  const int ntiles_rows = (rs.L + kRows - 1) / kRows;
  const int tile = level_offset(level) +
                   (level_count(level, ntiles_rows) - 1 - (int)blockIdx.x) * level_period(level);
  const int t0 = tile * kRows;
  const int L = rs.L, K = rs.topk, C = rs.C;
  const int nlmk = L / C;
  const int t_last = min(t0 + kRows, L) - 1;
  const int n_cand = min(t_last / C, nlmk);  // candidates of the tile's last row
  const int n_lo = min(t0 / C, nlmk);        // candidates of its first row
  const int n_ltiles = (n_cand + kTile - 1) / kTile;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_smem, 1);
    mbar_init(&bars->q_tmem, kRowThreads);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->l_full[s], 2);  // the TMA's bytes + the masking operand
      mbar_init(&bars->l_empty[s], 1);
    }
    for (int i = 0; i < kSBufs; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->s_empty[i], kRowThreads);
    }
    mbar_init(&bars->seed_ready, kRowThreads);
    mbar_init(&bars->seed_full, 1);
    mbar_init(&bars->seed_read, kRowThreads);
    mbar_init(&bars->seed_done, 1);
    mbar_init(&bars->done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < kRows) {
    tail_s[threadIdx.x] = 0u;
    head_s[threadIdx.x] = 0u;
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_l);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Lay::kTmemCols);
    tmem_relinquish();
  }
  // Seeds: the chunks every row's top-k starts from.  On levels above 0 they
  // are the selection of the last row of the tile `offset` positions earlier,
  // used when it is a full, strictly ascending set of that row's candidates
  // (all of them are candidates of this tile's rows too).  Otherwise they are
  // the chunks 0 .. min(k, n) - 1, which is where a plain scan would start.
  if (warp == 0) {
    int ns = 0;
    if (n_ltiles > 0) {
      bool anchored = false;
      if (level > 0) {
        const int anchor_t = min((tile - level_offset(level)) * kRows + kRows - 1, L - 1);
        const int anchor_n = min(anchor_t / C, nlmk);
        const int32_t *arow = sel + ((size_t)bh * L + anchor_t) * K;
        bool good = true;
        for (int i = lane; i < K; i += 32) {
          const int c = arow[i];
          const int prev = i > 0 ? arow[i - 1] : -1;
          good = good && c > prev && c < anchor_n;
          seed_list[i] = c;
        }
        anchored = __all_sync(0xffffffffu, good);
      }
      if (anchored) {
        ns = K;
      } else {
        ns = min(K, n_cand);
        for (int i = lane; i < ns; i += 32) seed_list[i] = i;
      }
    }
    if (lane == 0) *nseed_slot = ns;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int ns = *nseed_slot;
  // every candidate a seed (a short prefix): nothing left to scan
  const int n_scan = ns < n_cand ? n_ltiles : 0;
  const uint32_t tmem = *tmem_slot;
  const uint32_t q_tmem = tmem + Lay::kQCol;
  const uint32_t bias_tmem = tmem + Lay::kBiasCol;
  const uint32_t s_tmem0 = tmem + Lay::kSCol;  // score tile sb at s_tmem0 + sb * kTile
  const uint32_t seed_tmem = s_tmem0 + (kSBufs - 1) * kTile;  // free until tile kSBufs - 1
  unsigned char *seed_stage = smem + Lay::l0 + (kStages - 1) * Lay::kLBytes;
  const int lrow0 = (b * rs.Hkv + hkv) * nlmk;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (n_ltiles > 0) {
      if (lane == 0) {
        mbar_expect_tx(&bars->q_smem, Lay::kQBytes);
        for (int kb = 0; kb < D / 64; ++kb)
          tma_load_2d(smem + Lay::l0 + kb * kRows * 128, &tm_q, &bars->q_smem, kb * 64, bh * L + t0);
      }
      // the ring holds the Q tile until the row threads have moved it to TMEM
      bool ok = __all_sync(0xffffffffu, mbar_wait(&bars->q_tmem, 0, abort_flag, lim));
      const __nv_bfloat16 negb = __float2bfloat16_rn(-1.0e30f);
      const uint32_t neg = (uint32_t)__bfloat16_as_ushort(negb);
      int issued = 0;
      int cur = 0;  // seeds below tile i's columns have been passed
      for (int i = 0; ok && i < n_scan; ++i) {
        const int s = i % kStages;
        bool w = true;
        if (i >= kStages) w = mbar_wait(&bars->l_empty[s], ((i / kStages) - 1) & 1, abort_flag, lim);
        // the seed tile sits in the last ring stage until the seed MMA is done
        if (w && i == kStages - 1) w = mbar_wait(&bars->seed_done, 0, abort_flag, lim);
        if (!__all_sync(0xffffffffu, w)) break;
        // the landmark tile first (arrival 1 of 2, with its bytes) ...
        if (lane == 0) {
          mbar_expect_tx(&bars->l_full[s], Lay::kLBytes);
          unsigned char *ls = smem + Lay::l0 + s * Lay::kLBytes;
          for (int kb = 0; kb < D / 64; ++kb)
            tma_load_2d(ls + kb * kTile * 128, &tm_l, &bars->l_full[s], kb * 64, lrow0 + i * kTile);
        }
        ++issued;
        // ... then, while it is in flight, the seeds among its columns (the
        // ascending seed list walked 32 entries at a time) ...
        const int c0 = i * kTile;
        uint32_t m_lo = 0u, m_hi = 0u;
        for (;;) {
          const int idx = cur + lane;
          const int c = idx < ns ? seed_list[idx] : INT_MAX;
          const bool in = c < c0 + kTile;
          const uint32_t bal = __ballot_sync(0xffffffffu, in);
          const int rel = c - c0;
          m_lo |= __reduce_or_sync(0xffffffffu, in && rel < 32 ? (1u << rel) : 0u);
          m_hi |= __reduce_or_sync(0xffffffffu, in && rel >= 32 ? (1u << (rel - 32)) : 0u);
          cur += __popc(bal);
          if (bal != 0xffffffffu) break;
        }
        // ... and, for a tile that holds seeds or the row boundary (the last
        // one), its masking operand, K-slice s of the swizzled bias tile:
        // element 0 = -1e30 for seeds and columns past the candidates,
        // element 1 = -1e30 for the boundary chunk (first 64 rows only)
        const bool need = (m_lo | m_hi) != 0u || i == n_ltiles - 1;
        if (need) {
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int rr = lane + 32 * u;
            const int c = c0 + rr;
            const bool seed = ((u ? m_hi : m_lo) >> lane) & 1u;
            const uint32_t e0 = (seed || c >= n_cand) ? neg : 0u;
            const uint32_t e1 = (c == n_lo) ? neg : 0u;
            unsigned char *row = smem + Lay::bias + (rr >> 3) * 1024 + (rr & 7) * 128;
            *reinterpret_cast<uint4 *>(row + (((2 * s) ^ (rr & 7)) << 4)) = make_uint4(e0 | (e1 << 16), 0u, 0u, 0u);
            *reinterpret_cast<uint4 *>(row + (((2 * s + 1) ^ (rr & 7)) << 4)) = make_uint4(0u, 0u, 0u, 0u);
          }
          fence_async_smem();
        }
        __syncwarp();
        if (lane == 0) {
          bias_flag[s] = need ? 1 : 0;
          // arrival 2 of 2 (a failure-path test keeps back tile 0's: the MMA
          // issuer's bounded wait then runs out and every role unwinds)
          if (!(rs.withhold && i == 0)) mbar_arrive(&bars->l_full[s]);
        }
      }
      if (lane == 0) {
        for (int i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
          mbar_wait_bounded(&bars->l_full[i % kStages], (i / kStages) & 1, lim);
        mbar_wait_bounded(&bars->q_smem, 0, lim);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_ltiles > 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kRows, kTile, false, false);
      bool ok = mbar_wait(&bars->q_tmem, 0, abort_flag, lim);
      // seed scores: Q * seeds^T (the seed landmark rows, staged by the rows)
      ok = ok && mbar_wait(&bars->seed_ready, 0, abort_flag, lim);
      tc_fence_after();
      if (ok) {
        const uint32_t sd_addr = smem_u32(seed_stage);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int kb = kk >> 2, kw = kk & 3;
          const uint64_t bd = smem_desc_sw128(sd_addr + kb * kTile * 128 + kw * 32, 16, 1024);
          mma_bf16_ts(seed_tmem, q_tmem + kk * 8, bd, idesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars->seed_full);
        mma_commit(&bars->seed_done);
      }
      const uint32_t bias_addr = smem_u32(smem + Lay::bias);
      for (int i = 0; ok && i < n_scan; ++i) {
        const int s = i % kStages, sb = i % kSBufs;
        if (!mbar_wait(&bars->l_full[s], (i / kStages) & 1, abort_flag, lim)) break;
        if (i >= kSBufs && !mbar_wait(&bars->s_empty[sb], ((i / kSBufs) - 1) & 1, abort_flag, lim)) break;
        if (i == kSBufs - 1 && !mbar_wait(&bars->seed_read, 0, abort_flag, lim)) break;
        tc_fence_after();
        const uint32_t l_addr = smem_u32(smem + Lay::l0 + s * Lay::kLBytes);
        const uint32_t d_tmem = s_tmem0 + sb * kTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int kb = kk >> 2, kw = kk & 3;
          const uint64_t bd = smem_desc_sw128(l_addr + kb * kTile * 128 + kw * 32, 16, 1024);
          mma_bf16_ts(d_tmem, q_tmem + kk * 8, bd, idesc, kk > 0 ? 1u : 0u);
        }
        // the masking step, on tiles that need one: S += [1, row < 64] * bias_s^T
        if (bias_flag[s])
          mma_bf16_ts(d_tmem, bias_tmem, smem_desc_sw128(bias_addr + s * 32, 16, 1024), idesc, 1u);
        mma_commit(&bars->s_full[sb]);
        mma_commit(&bars->l_empty[s]);
      }
      mma_commit(&bars->done);
      mbar_wait_bounded(&bars->done, 0, lim);
    }
  } else {
    // ---------------------------------------------------------- row threads
    const int h = (warp - 2) >> 2;         // 0: owner, columns [0, 32); 1: columns [32, 64)
    const int r = 32 * (warp & 3) + lane;  // TMEM lane == tile row
    const int rt = r + kRows * h;
    const int t = t0 + r;
    const bool valid = t < L;
    const int n_c = valid ? min(t / C, nlmk) : 0;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    uint64_t *slots = reinterpret_cast<uint64_t *>(smem + Lay::heap) + r;
    uint64_t *mbox = reinterpret_cast<uint64_t *>(smem + Lay::mbox) + r;
    const float c2 = rs.scale * kLog2e;
    const float sc = rs.scale;
    const float inv_sc = 1.0f / sc;
    const bool want_lse = lse_lmk != nullptr;
    float m2 = -INFINITY, l = 0.0f;
    // rows with at most k candidates keep all of them (no search); with
    // seeds, the first `cnt` seeds are the row's starting set (all of them
    // are candidates of the row)
    const int cnt = n_c <= K ? n_c : K;
    const bool search = n_c > K;
    TopK tk;
    tk.thr = INFINITY;
    tk.mn = ~0ull;
    tk.mg = 0;
    tk.gpos = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) tk.gmin[i] = ~0ull;
    bool ok = true;
    if (n_ltiles > 0) {
      // q row -> tensor memory (A operand of the scoring MMA): the row's
      // 128-byte lines of the swizzled staging tile, two bf16 per column;
      // the owner also writes the masking operand [1, row < 64, 0, ...]
      ok = mbar_wait(&bars->q_smem, 0, abort_flag, lim);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        if (hp.npairs > 0) {
          // HoPE on the fly: the query rotated as the pre-pass would
          hope_row_split<D>(smem + Lay::l0, r, h, hp, (long long)hp.pos0 + t, q_tmem + lane_off);
        } else if (h < D / 64) {
          uint32_t w[32];
          const unsigned char *line = smem + Lay::l0 + h * kRows * 128 + r * 128;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint4 v4 = *reinterpret_cast<const uint4 *>(line + ((j ^ (r & 7)) << 4));
            w[4 * j] = v4.x;
            w[4 * j + 1] = v4.y;
            w[4 * j + 2] = v4.z;
            w[4 * j + 3] = v4.w;
          }
          tmem_st32(q_tmem + lane_off + h * 32, w);
        }
        if (h == 0) {
          const __nv_bfloat162 p01 = __floats2bfloat162_rn(1.0f, r < kTile ? 1.0f : 0.0f);
          uint32_t w8[8] = {*reinterpret_cast<const uint32_t *>(&p01), 0u, 0u, 0u, 0u, 0u, 0u, 0u};
          tmem_st8(bias_tmem + lane_off, w8);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(&bars->q_tmem);
      // stage the seed landmark rows into the last ring stage (128-byte
      // swizzled, as a TMA tile would be) once every row has read its Q
      // line out of it; rows past the seed count are zero
      rows_sync();
      if (ok) {
        constexpr int kPieces = D / 8;  // 16-byte pieces per row
#pragma unroll 1
        for (int pc = rt; pc < kTile * kPieces; pc += kRowThreads) {
          const int sr = pc / kPieces, col = pc % kPieces, kb = col >> 3, j = col & 7;
          uint4 v4 = make_uint4(0u, 0u, 0u, 0u);
          if (sr < ns)
            v4 = *reinterpret_cast<const uint4 *>(
                reinterpret_cast<const unsigned char *>(lmk_raw) +
                ((size_t)(lrow0 + seed_list[sr]) * D + kb * 64 + j * 8) * 2);
          *reinterpret_cast<uint4 *>(seed_stage + kb * kTile * 128 + sr * 128 +
                                     ((j ^ (sr & 7)) << 4)) = v4;
        }
      }
      fence_async_smem();
      mbar_arrive(&bars->seed_ready);
      ok = __all_sync(0xffffffffu, ok && mbar_wait(&bars->seed_full, 0, abort_flag, lim));
      if (ok) {
        tc_fence_after();
        float sa[32];
        tmem_ld32(seed_tmem + lane_off + 32 * h, sa);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&bars->seed_read);
        // this thread's half of the starting set, and its log-sum-exp
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int jj = 32 * h + j;
          if (jj < cnt) slots[jj * kRows] = sel_key(sa[j] * sc, seed_list[jj]);
          sa[j] = jj < cnt ? sa[j] : -INFINITY;
        }
        if (want_lse) {
          const float bm = block_max(sa);
          if (bm > -INFINITY) lse_block(sa, bm, c2, m2, l);
        }
      }
    }
    rows_sync();  // both halves of every row's starting set are in place
    if (h == 0) {
      if (ok && search) tk.build(slots, K);
      st_volf(&thr_s[r], prefilter(tk.thr, inv_sc));
    }
    rows_sync();
    float thr_u = thr_s[r];
    uint32_t mb = 0;  // owner: keys drained; other half: keys posted
    // owner: insert what the other half posted so far; returns the raw tail
    auto drain = [&]() -> uint32_t {
      const uint32_t tv = ld_vol(&tail_s[r]);
      const uint32_t tl = tv & ~kDone;
      while (mb != tl) {
        __threadfence_block();
        const uint64_t key = reinterpret_cast<volatile uint64_t *>(mbox)[(mb % kMbox) * kRows];
        ++mb;
        __threadfence_block();
        st_vol(&head_s[r], mb);
        if (key > tk.mn) {
          tk.replace(slots, key, K);
          thr_u = prefilter(tk.thr, inv_sc);
          st_volf(&thr_s[r], thr_u);
        }
      }
      return tv;
    };
    for (int i = 0; ok && i < n_scan; ++i) {
      const int sb = i % kSBufs;
      const uint32_t par = (i / kSBufs) & 1;
      if (h == 0) {
        // The owner keeps draining while it waits: the other half may be a
        // tile behind, waiting for mailbox room, and the next score tile
        // needs that half to release the one before.
        bool got = mbar_try_wait(&bars->s_full[sb], par);
        if (!got) {
          const uint64_t w0 = globaltimer();
          for (uint32_t it = 1;; ++it) {
            drain();
            if (mbar_try_wait(&bars->s_full[sb], par)) { got = true; break; }
            if ((it & 63u) == 0) {
              if (*abort_flag) break;
              if (globaltimer() - w0 > lim) { *abort_flag = 1; break; }
            }
          }
        }
        ok = got;
      } else {
        ok = mbar_wait(&bars->s_full[sb], par, abort_flag, lim);
      }
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      float a[32];
      tmem_ld32(s_tmem0 + sb * kTile + lane_off + 32 * h, a);
      if (h == 0)
        drain();  // the other half's candidates since the last tile
      else
        thr_u = ld_volf(&thr_s[r]);
      __syncwarp();  // tcgen05.wait is warp-collective
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bars->s_empty[sb]);
      const int cb = i * kTile + 32 * h;
      const float bm = block_max(a);
      if (want_lse) lse_block(a, bm, c2, m2, l);
      // candidates that may enter the top-k (seeds and masked columns sit at -1e30)
      const bool pass = bm >= thr_u;
      if (!__any_sync(0xffffffffu, pass)) continue;
      uint32_t mask = pass ? ge_mask(a, thr_u) : 0u;
      const bool single = __popc(mask) == 1;  // then it is the block maximum
      // one candidate per lane per iteration: the lanes insert together
      while (__any_sync(0xffffffffu, mask != 0)) {
        if (mask) {
          const int j = __ffs(mask) - 1;
          mask &= mask - 1;
          const float v = single ? bm : pick32(a, j);
          const uint64_t key = sel_key(v * sc, cb + j);
          if (h == 0) {
            if (key > tk.mn) {
              tk.replace(slots, key, K);
              thr_u = prefilter(tk.thr, inv_sc);
              st_volf(&thr_s[r], thr_u);
            }
          } else {
            // wait (bounded) for a free mailbox entry, then post
            bool room = mb - ld_vol(&head_s[r]) < (uint32_t)kMbox;
            if (!room) {
              const uint64_t w0 = globaltimer();
              while (!room) {
                if (*abort_flag || globaltimer() - w0 > lim) break;
                room = mb - ld_vol(&head_s[r]) < (uint32_t)kMbox;
              }
            }
            if (!room) {
              *abort_flag = 1;
              ok = false;
              mask = 0;
            } else {
              __threadfence_block();
              reinterpret_cast<volatile uint64_t *>(mbox)[(mb % kMbox) * kRows] = key;
              ++mb;
              __threadfence_block();
              st_vol(&tail_s[r], mb);
            }
          }
        }
      }
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
    }
    if (h == 1) {
      // hand over this half's log-sum-exp and close the mailbox
      lsep_s[r] = make_float2(m2, l);
      __threadfence_block();
      st_vol(&tail_s[r], mb | kDone);
    } else {
      // drain what the other half still posts until it closes the mailbox
      const uint64_t w0 = globaltimer();
      bool closed = false;
      for (uint32_t it = 0;; ++it) {
        const uint32_t tv = drain();
        if ((tv & kDone) && mb == (tv & ~kDone)) { closed = true; break; }
        if ((it & 63u) == 63u && (globaltimer() - w0 > lim)) break;
      }
      if (!closed) {
        *abort_flag = 1;
        ok = false;
      }
      __threadfence_block();
      // ---------------------------------------------------------- epilogue
      if constexpr (Lay::kStagedOut) {
        // The warp's rows are 32 consecutive positions inside one chunk, so
        // every valid lane has the candidate count of the warp's first row
        // and the choice of the staged path is uniform over the warp (lanes
        // past L take part but write nothing).  The staging blocks (K = 32
        // or 64) sit in the landmark ring and the masking tile, idle once
        // this warp has read its last score tile.
        const size_t row = (size_t)bh * L + t;
        const int wrow0 = t0 + 32 * (warp & 3);  // the warp's first position
        const int rows_valid = min(32, L - wrow0);
        const int n_c_warp = min(wrow0 / C, nlmk);
        if (__all_sync(0xffffffffu, ok) && rows_valid > 0 && n_c_warp > K && (K == 64 || K == 32)) {
          uint32_t *stage = reinterpret_cast<uint32_t *>(smem + Lay::l0) + (warp & 3) * 32 * (K + 4);
          const size_t r0 = (size_t)bh * L + wrow0;
          if (K == 64)
            write_sorted_staged<64>(slots, stage, lane, sel + r0 * K, chunk_w + r0 * K, rows_valid);
          else
            write_sorted_staged<32>(slots, stage, lane, sel + r0 * K, chunk_w + r0 * K, rows_valid);
        } else if (__all_sync(0xffffffffu, ok) && valid) {
          write_row(slots, n_c, cnt, K, sel + row * K, chunk_w + row * K);
        }
        if (__all_sync(0xffffffffu, ok) && valid && want_lse)
          lse_lmk[row] = row_lse(lsep_s[r], m2, l, n_c);
      } else {
        if (__all_sync(0xffffffffu, ok) && valid) {
          const size_t row = (size_t)bh * L + t;
          write_row(slots, n_c, cnt, K, sel + row * K, chunk_w + row * K);
          if (want_lse) lse_lmk[row] = row_lse(lsep_s[r], m2, l, n_c);
        }
      }
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
                         float *w, float *lse_lmk, uint32_t *err, cudaStream_t st,
                         int *launches, const HopeParams &hp) {
  CUtensorMap tq, tl;
  cudaError_t e;
  const int nlmk = rs.L / rs.C;
  const uint64_t qrows = (uint64_t)rs.B * rs.Hq * rs.L;
  const uint64_t lrows = (uint64_t)rs.B * rs.Hkv * (nlmk > 0 ? nlmk : 1);
  if ((e = make_tmap_bf16(&tq, q, qrows, rs.d, kRows)) != cudaSuccess) return e;
  // with no complete chunk the landmark map is never read; point it at q
  if ((e = make_tmap_bf16(&tl, nlmk > 0 ? lmk : q, lrows, rs.d, kTile)) != cudaSuccess) return e;
  const int ntiles = (rs.L + kRows - 1) / kRows;
  const __nv_bfloat16 *lraw = static_cast<const __nv_bfloat16 *>(lmk);
  auto launch = [&](auto kern, size_t smem) -> cudaError_t {
    cudaError_t e2 = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e2 != cudaSuccess) return e2;
    for (int lv = 0; lv < kLevels; ++lv) {
      const int n = level_count(lv, ntiles);
      if (n == 0) continue;
      kern<<<dim3(n, rs.B * rs.Hq), kThreads, smem, st>>>(tq, tl, rs, sel, w, lse_lmk, err, lv, lraw, hp);
      ++*launches;
      if ((e2 = cudaGetLastError()) != cudaSuccess) return e2;
    }
    return cudaSuccess;
  };
  if (rs.d == 64) return launch(select_sm100_kernel<64>, SelLayout<64>::total);
  return launch(select_sm100_kernel<128>, SelLayout<128>::total);
}

}  // namespace hils
