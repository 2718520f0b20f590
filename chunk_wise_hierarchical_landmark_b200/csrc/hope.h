// HoPE pre-pass (declaration shared by the C ABI and hope.cu).
#pragma once

#include <cuda_runtime.h>

namespace hils {

// Rotate, in place, the first n_rope_pairs rotate-half pairs of every row of
// x [BH][L][d] (fp32 or bf16) by the angle (pos0 + t) * base^(-2i/d).
cudaError_t hope_apply(void *x, bool bf16, int BH, int L, int d, int pos0, int n_rope_pairs,
                       double base, cudaStream_t st, int *launches);

}  // namespace hils
