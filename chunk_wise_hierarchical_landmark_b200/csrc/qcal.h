// Q-Cal scoring query kernels (qcal.cu).
#pragma once

#include <cuda_runtime.h>

namespace hils {

constexpr int kMaxQcalRank = 64;  // largest rank r of the low-rank offset

// q_cal = q + W_up[hq] (W_down h) for every (b, hq, t), rounded to the query
// dtype; z [B, L, r] fp32 is scratch.  Two launches.
cudaError_t qcal_query(bool bf16, int B, int Hq, int L, int d, int D, int r, const void *q,
                       const void *h, const void *w_down, const void *w_up, void *q_cal,
                       float *z, cudaStream_t st, int *launches);

}  // namespace hils
