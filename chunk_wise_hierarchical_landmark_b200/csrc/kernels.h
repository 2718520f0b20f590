// Internal launcher interface between the C-ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "hope.cuh"

namespace hils {

// Rows handled by a launch: positions [t_first, t_first + t_count) of every
// (b, hq) head.  Query row (bh, t) lives at q + (bh * t_count + t - t_first) * d
// and so do the per-row outputs (prefill: t_first = 0, t_count = L; decode:
// t_first = N - 1, t_count = 1 with q laid out [B, Hq, d]).
struct RowSpec {
  int B, Hq, Hkv, L, d, C, topk;
  float scale;
  int t_first, t_count;
  // bounded device waits give up after wait_ns; withhold = 1 (tests of the
  // failure path only) keeps back one producer arrival of the scoring kernel
  unsigned long long wait_ns = 2000000000ull;
  int withhold = 0;
};

// SIMT kernels (hils_simt.cu)
cudaError_t select_simt(const RowSpec &rs, bool bf16, const void *q, const void *lmk,
                        int32_t *sel, float *w, float *lse_lmk, cudaStream_t st);
cudaError_t attn_simt(const RowSpec &rs, bool bf16, const void *q, const void *k, const void *v,
                      const int32_t *sel, const float *w, void *out, float *lse, float *wfin,
                      uint32_t *err, cudaStream_t st);
size_t simt_attn_smem(int d, int L, int C);

// tcgen05 attention for bf16 prefill (attn_sm100.cu)
// hp: HoPE applied to the query tile on the fly (hp.npairs = 0: none)
cudaError_t attn_sm100(const RowSpec &rs, const void *q, const void *k, const void *v,
                       const int32_t *sel, const float *w, void *out, float *lse, float *wfin,
                       uint32_t *err, cudaStream_t st, const HopeParams &hp);
size_t attn_sm100_smem(int d, int L);

// tcgen05 landmark scoring + top-k for bf16 prefill (select_sm100.cu)
cudaError_t select_sm100(const RowSpec &rs, const void *q, const void *lmk, int32_t *sel,
                         float *w, float *lse_lmk, uint32_t *err, cudaStream_t st,
                         int *launches, const HopeParams &hp);

}  // namespace hils

#include <cuda.h>
namespace hils {
// 2-D bf16 TMA descriptor over a row-major [rows, cols] array: box
// [box_rows x 64 elements], 128-byte swizzle (attn_sm100.cu)
cudaError_t make_tmap_bf16(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                           uint32_t box_rows);
// the same over an fp32 array: box [box_rows x 32 elements] (128 bytes)
cudaError_t make_tmap_f32(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                          uint32_t box_rows);

// Decode step (decode.cu).  One query per head at position N-1.
struct DecodeSpec {
  int B, Hq, Hkv, N, d, topk;
  float scale;
  int own, nlmk, n_c;  // own chunk, landmark rows per KV head, completed chunks
  int P;               // landmark slabs of 256 (scoring CTAs per KV head)
  int nwords;          // chunk bitmap words
  int ucap;            // union capacity per KV head: G * topk + 1
  int Q;               // attention CTAs per KV head
};
DecodeSpec decode_spec(int B, int Hq, int Hkv, int N, int d, int topk, float scale);
size_t decode_workspace_bytes(const DecodeSpec &ds);
size_t decode_max_g();
cudaError_t decode_fwd(const DecodeSpec &ds, bool bf16, const void *q, const void *k,
                       const void *v, const void *lmk, int32_t *sel, float *w, float *lse_lmk,
                       void *out, float *lse, void *ws, uint32_t *err, cudaStream_t st,
                       int *launches);

// Internal (not exported): set the calling thread's hils_last_error() text.
extern "C" void hils_internal_set_error(const char *msg);

// Chunk union in CSR form (hils_union.cu)
cudaError_t union_csr(int B, int Hq, int L, int C, int topk, int M, const int32_t *sel,
                      int32_t *u_off, int32_t *u_idx, int64_t u_cap, uint32_t *err,
                      cudaStream_t st, int *launches);

}  // namespace hils
