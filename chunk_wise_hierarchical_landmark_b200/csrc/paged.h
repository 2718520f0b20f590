// Decode step over a paged KV cache (declarations shared by the C ABI and
// decode.cu).
#pragma once

#include "kernels.h"

namespace hils {

// Paged K/V: page = one chunk of C tokens of every KV head, pools
// [num_pages][Hkv][C][d]; table[b * max_pages + c] is the page of chunk c of
// sequence b.
struct PagedKV {
  const int32_t *table;
  int max_pages;
  long long num_pages;
};

// decode_fwd with K and V read through the page table (the landmark keys
// stay dense [B][Hkv][N/C][d]).
cudaError_t decode_fwd_paged(const DecodeSpec &ds, bool bf16, const void *q, const void *k_pages,
                             const void *v_pages, const PagedKV &pages, const void *lmk,
                             int32_t *sel, float *w, float *lse_lmk, void *out, float *lse,
                             void *ws, uint32_t *err, cudaStream_t st, int *launches);

}  // namespace hils
