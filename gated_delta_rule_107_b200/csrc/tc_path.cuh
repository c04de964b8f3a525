// tc_path.cuh -- the tcgen05 tensor-core path (bf16 I/O, dk = dv = 128, chunk 64).
#pragma once
#include "dr_common.cuh"

namespace dr {

bool tc_fwd_supported(const Geo &g, bool bf16);
size_t tc_fwd_ws_bytes(const Geo &g);
cudaError_t tc_fwd(const Geo &g, const Tensors &t, void *workspace, cudaStream_t s, Rec &rec);
// warp-specialised forward for Gated DeltaNet / DeltaNet (tc_fwd2.cu)
cudaError_t tc_fwd2(const Geo &g, const Tensors &t, cudaStream_t s, Rec &rec);
// Workspace of the tensor-core backward, chunk-major (ci = (b H + h) N + n), every
// matrix row-major: bf16 tiles the gradient kernel loads with TMA, plus the fp32 gate.
struct TcBwdWs {
    __nv_bfloat16 *Sn;   // [ci][dk][dv]  state entering chunk n
    __nv_bfloat16 *dSn;  // [ci][dk][dv]  dL/dS of the state leaving chunk n
    __nv_bfloat16 *Un;   // [ci][C][dv]   write values U = U~ - W S_n
    __nv_bfloat16 *W;    // [ci][C][dk]   W  = T diag(beta e^g) k
    __nv_bfloat16 *Ut;   // [ci][C][dv]   U~ = T diag(beta) v
    __nv_bfloat16 *P;    // [ci][C][C]    P  = tril(e^{g_r - g_i} q_r . k_i)
    __nv_bfloat16 *Tn;   // [ci][C][C]    T  = (I + A)^-1
    __nv_bfloat16 *KK;   // [ci][C][C]    k k^T (no gate factor)
    float *g;            // [ci][C]       in-chunk cumulative log gate
};
size_t tc_bwd_ws_bytes(const Geo &g);
TcBwdWs tc_bwd_ws_carve(const Geo &g, void *base);
// Gated DeltaNet / DeltaNet, bf16, dk = dv = 128, C = 64, and chunk row indices that fit
// the 32-bit coordinates of a TMA load.
bool tc_bwd_recompute_supported(const Geo &g, bool bf16);
// Backward recompute (tc_fwd2.cu, recompute mode): fills g, KK, P, T, W, U~, S_n and U.
cudaError_t tc_bwd_recompute(const Geo &g, const Tensors &t, const TcBwdWs &w, cudaStream_t s, Rec &rec);
// Reverse state chain (tc_fwd2.cu, reverse mode): dS_{n+1} of every chunk into w.dSn, and dS0.
cudaError_t tc_bwd_reverse(const Geo &g, const Tensors &t, const TcBwdWs &w, cudaStream_t s, Rec &rec);
// All intra-chunk gradients (tc_bwd.cu): dq, dk, dv, dbeta, d log alpha.
cudaError_t tc_bwd_chunk(const Geo &g, const Tensors &t, const TcBwdWs &w, cudaStream_t s, Rec &rec);
// number of launches of tc_fwd and their names
int tc_fwd_launches(const Geo &g, const char **names, int max_names);

}  // namespace dr
