// Backward pass kernels (backward.cu).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace hils {

struct BwdSpec {
  int B, Hq, Hkv, L, d, topk;
  float scale;
  int nch;   // chunks of a sequence (the last may be partial)
  int nlmk;  // landmark rows per KV head (complete chunks)
};
BwdSpec bwd_spec(int B, int Hq, int Hkv, int L, int d, int topk, float scale);
size_t bwd_workspace_bytes(const BwdSpec &bs);
cudaError_t bwd_run(const BwdSpec &bs, bool bf16, const void *q, const void *k, const void *v,
                    const void *lmk, const int32_t *sel, const float *chunk_w, const float *lse,
                    const void *dout, const float *dlse, float *dq, float *dk, float *dv,
                    float *dlmk, void *ws, uint32_t *err, cudaStream_t st, int *launches);

}  // namespace hils
