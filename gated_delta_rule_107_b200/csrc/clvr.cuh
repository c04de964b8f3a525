// clvr.cuh -- cross-layer value routing (clvr.cu).
#pragma once
#include "dr_common.cuh"

namespace dr {

size_t clvr_ws_bytes();
// h_out [M][N] = h + U W (h NULL: zero); U [M][K], W [K][N]; all in the I/O dtype
int clvr_fwd_run(const void *U, const void *W, const void *h, void *h_out, int M, int K, int N, bool bf16,
                 void *ws, size_t ws_bytes, cudaStream_t s);
// dU [M][K] = dH W^T (I/O dtype; NULL = skip), dW [K][N] = U^T dH (fp32; NULL = skip)
int clvr_bwd_run(const void *U, const void *W, const void *dH, void *dU, float *dW, int M, int K, int N, bool bf16,
                 void *ws, size_t ws_bytes, cudaStream_t s);

}  // namespace dr
