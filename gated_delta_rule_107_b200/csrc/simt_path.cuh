// simt_path.cuh -- the fp32 CUDA-core path (any supported shape, fp32 or bf16 I/O).
#pragma once
#include "dr_common.cuh"

namespace dr {

// fp32 workspace of the CUDA-core path, chunk-major.  C = chunk, N = chunks.
struct SimtWs {
    float *W;    // [B,H,N,C,dk]  W  = (I+A)^-1 diag(beta) Ktil
    float *Ut;   // [B,H,N,C,dv]  U~ = (I+A)^-1 diag(beta) V
    float *G;    // [B,H,N,C,dk]  in-chunk cumulative log gate g (per channel)
    float *P;    // [B,H,N,C,C]   P  = tril(Qtil Khat^T)
    float *Sn;   // [B,H,N,dk,dv] state entering chunk n
    float *Un;   // [B,H,N,C,dv]  write values U = U~ - W S
    // backward only
    float *dSn;  // [B,H,N,dk,dv] dL/dS for the state leaving chunk n
    float *dUn;  // [B,H,N,C,dv]  total dL/dU
    float *Qd;   // [B,H,N,C,dk]  dO S^T
    float *dWm;  // [B,H,N,C,dk]  -dU S^T   (= dL/dW)
    float *Tm;   // [B,H,N,C,dk]  U dS+^T
    float *RS;   // [B,H,N,dk]    rowsum(S .* dS+)
    const int *only;  // optional [B,H,N]: the intra-chunk gradient kernel serves the flagged chunks alone
};

size_t simt_ws_bytes(const Geo &g, bool bwd);
SimtWs simt_ws_carve(const Geo &g, bool bwd, void *base);
cudaError_t simt_fwd(const Geo &g, const Tensors &t, bool bf16, const SimtWs &w, cudaStream_t s, Rec &rec);
cudaError_t simt_bwd(const Geo &g, const Tensors &t, bool bf16, const SimtWs &w, cudaStream_t s, Rec &rec);
// The backward's last two kernels (k_bwd_state, k_bwd_intra), for a w whose G, W, Ut, P, Sn,
// Un hold the forward's values and dSn, dUn the reverse chain's (from tensor-core kernels).
cudaError_t simt_bwd_grads(const Geo &g, const Tensors &t, bool bf16, const SimtWs &w, cudaStream_t s, Rec &rec);
// The intra-chunk gradient kernel alone: w holds, besides what simt_bwd_grads reads, the
// state products Qd, dWm, Tm, RS.
cudaError_t simt_bwd_intra(const Geo &g, const Tensors &t, bool bf16, const SimtWs &w, cudaStream_t s, Rec &rec);
// kernel names in launch order (for the timed entry points)
extern const char *const SIMT_FWD_KERNELS[3];
extern const char *const SIMT_BWD_KERNELS[5];

}  // namespace dr
