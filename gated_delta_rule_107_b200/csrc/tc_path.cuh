// tc_path.cuh -- the tcgen05 tensor-core path (bf16 I/O, dk = 128, chunk 64).
//
// Gated DeltaNet and DeltaNet at dv = 128 run the split path: a per-chunk kernel over all
// chunks at once (tc_prep.cu), the serial state chains (tc_chain.cu) and, for the
// backward, the per-chunk gradient kernel (tc_bwd.cu).  KDA and dv = 64 run the
// single-kernel forward of tc_fwd.cu.
#pragma once
#include "dr_common.cuh"

namespace dr {

bool tc_fwd_supported(const Geo &g, bool bf16);
cudaError_t tc_fwd(const Geo &g, const Tensors &t, void *workspace, cudaStream_t s, Rec &rec);
// number of launches of tc_fwd and their names
int tc_fwd_launches(const Geo &g, const char **names, int max_names);

// Split path: Gated DeltaNet / DeltaNet, bf16, dk = dv = 128, C = 64, and chunk row
// indices that fit the 32-bit coordinates of a TMA load.
bool tc_split_supported(const Geo &g, bool bf16);

// Workspace of the split path, chunk-major (ci = (b H + h) N + n), every matrix row-major:
// bf16 tiles that later kernels load with TMA, plus fp32 per-token factors.  The forward
// uses gb, W, Ut and P; the backward all of it.
struct TcWs {
    float *gb;           // [ci][2][C]    in-chunk cumulative log gate g, then beta
    __nv_bfloat16 *W;    // [ci][C][dk]   W  = T diag(beta e^g) k
    __nv_bfloat16 *Ut;   // [ci][C][dv]   U~ = T diag(beta) v
    __nv_bfloat16 *P;    // [ci][C][C]    P  = tril(e^{g_r - g_i} q_r . k_i)
    // backward only
    __nv_bfloat16 *Tn;   // [ci][C][C]    T  = (I + A)^-1
    __nv_bfloat16 *KK;   // [ci][C][C]    k k^T (no gate factor)
    __nv_bfloat16 *dUp;  // [ci][C][dv]   P^T dO
    __nv_bfloat16 *Sn;   // [ci][dk][dv]  state entering chunk n
    __nv_bfloat16 *dSn;  // [ci][dk][dv]  dL/dS of the state leaving chunk n
    __nv_bfloat16 *Un;   // [ci][C][dv]   write values U = U~ - W S_n
    __nv_bfloat16 *dUn;  // [ci][C][dv]   dL/dU = du + P^T dO + Kbar dS_{n+1}
    float *skt;          // [ci][2][C]    per 64-column half of dv: U_r . (Kbar dS_{n+1})_r
};
size_t tc_ws_bytes(const Geo &g, bool bwd);
TcWs tc_ws_carve(const Geo &g, bool bwd, void *base);

// Per-chunk products (tc_prep.cu): g and beta, W, U~, P; with bwd also T, k k^T and P^T dO.
cudaError_t tc_chunk_prep(const Geo &g, const Tensors &t, const TcWs &w, bool bwd, cudaStream_t s, Rec &rec);
// Forward state chain (tc_chain.cu).  bwd = false: o, u, S_T; bwd = true (recompute for the
// backward): S_n and U of every chunk into the workspace.
cudaError_t tc_chain_fwd(const Geo &g, const Tensors &t, const TcWs &w, bool bwd, cudaStream_t s, Rec &rec);
// Reverse state chain (tc_chain.cu): dS_{n+1} and dL/dU of every chunk (w.dSn, w.dUn), the
// row sums w.skt, and dS0.
cudaError_t tc_chain_rev(const Geo &g, const Tensors &t, const TcWs &w, cudaStream_t s, Rec &rec);
// All intra-chunk gradients (tc_bwd.cu): dq, dk, dv, dbeta, d log alpha.
cudaError_t tc_bwd_chunk(const Geo &g, const Tensors &t, const TcWs &w, cudaStream_t s, Rec &rec);

}  // namespace dr
