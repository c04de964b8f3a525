// decode.cuh -- the recurrent (token-by-token) forward for short sequences (decode.cu).
#pragma once
#include "dr_common.cuh"

namespace dr {
// t.S0 (null = zero) -> t.S_T (null = not written; may equal t.S0); writes t.out, t.u.
cudaError_t decode_fwd(const Geo &g, const Tensors &t, bool bf16, cudaStream_t s, Rec &rec);
}  // namespace dr
