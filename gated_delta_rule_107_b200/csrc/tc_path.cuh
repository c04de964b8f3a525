// tc_path.cuh -- the tcgen05 tensor-core path (bf16 I/O, dk = 128, chunk 64).
//
// Gated DeltaNet and DeltaNet at dv = 128 run the split path: a per-chunk kernel over all
// chunks at once (tc_prep.cu), the serial state chains (tc_chain.cu) and, for the
// backward, the per-chunk gradient kernel (tc_bwd.cu); api.cu sequences them.  KDA and
// dv = 64 run the single-kernel forward of tc_fwd.cu.
#pragma once
#include "dr_common.cuh"

namespace dr {

bool tc_fwd_supported(const Geo &g, bool bf16);
// the single-kernel forward (KDA, and Gated DeltaNet / DeltaNet at dv = 64); no workspace
cudaError_t tc_fwd(const Geo &g, const Tensors &t, void *workspace, cudaStream_t s, Rec &rec);
// number of launches of tc_fwd and their names
int tc_fwd_launches(const Geo &g, const char **names, int max_names);

// Split path: Gated DeltaNet / DeltaNet, bf16, dk = dv = 128, C = 64, and chunk row
// indices that fit the 32-bit coordinates of a TMA load.
bool tc_split_supported(const Geo &g, bool bf16);
// The same shapes for KDA: the split forward (the backward stays on the CUDA-core path).
bool tc_split_kda_supported(const Geo &g, bool bf16);

// Workspace of the split path, chunk-major (ci = (b H + h) N + n), every matrix row-major:
// bf16 tiles that later kernels load with TMA, plus fp32 per-token factors.  Three parts:
//   WS_FWD   the forward's chunk products (gb, W, Ut, P);
//   WS_KEEP  what the backward needs from the forward besides them (Tn, KK, Sn, Un);
//   WS_REV   what the reverse chain hands the gradient kernel (dSn, dUn, skt).
// The forward's workspace is WS_FWD; the recomputing backward's all three; the saved
// activations of delta_rule_fwd_save are WS_FWD | WS_KEEP, and the backward from them needs
// WS_REV as workspace.
struct TcWs {
    float *gb;           // [ci][2][C]    in-chunk cumulative log gate g, then beta
    __nv_bfloat16 *W;    // [ci][C][dk]   W  = T diag(beta e^g) k
    __nv_bfloat16 *Ut;   // [ci][C][dv]   U~ = T diag(beta) v
    __nv_bfloat16 *P;    // [ci][C][C]    P  = tril(e^{g_r - g_i} q_r . k_i)
    __nv_bfloat16 *Tn;   // [ci][C][C]    T  = (I + A)^-1
    __nv_bfloat16 *KK;   // [ci][C][C]    k k^T (no gate factor)
    __nv_bfloat16 *Sn;   // [ci][dk][dv]  state entering chunk n
    __nv_bfloat16 *Un;   // [ci][C][dv]   write values U = U~ - W S_n
    __nv_bfloat16 *dSn;  // [ci][dk][dv]  dL/dS of the state leaving chunk n
    __nv_bfloat16 *dUn;  // [ci][C][dv]   dL/dU = du + P^T dO + Kbar dS_{n+1}
    float *skt;          // [ci][2][C]    per 64-column half of dv: U_r . (Kbar dS_{n+1})_r
    // KDA forward (channel-wise gates, g = in-chunk cumulative log gate per key channel,
    // g_m its value at the chunk's middle token, exponents clamped to [-80, 80]):
    __nv_bfloat16 *Kt1;  // [ci][C][dk]   k e^{g - g_m}      (rows of P1's A)
    __nv_bfloat16 *Qt1;  // [ci][C][dk]   q e^{g - g_m}      (rows of P1's A)
    __nv_bfloat16 *Kh;   // [ci][C][dk]   k e^{g_m - g}      (P1's B)
    __nv_bfloat16 *Kt;   // [ci][C][dk]   k e^{g}            (W = T diag(beta) Kt)
    __nv_bfloat16 *Qt;   // [ci][C][dk]   q e^{g}            (o = Qt S + P U)
    __nv_bfloat16 *Kb;   // [ci][C][dk]   k e^{g_C - g}      (S+ = Diag(e^{g_C}) S + Kb^T U)
    float *egc;          // [ci][dk]      e^{g_C}
};
enum { WS_FWD = 1, WS_KEEP = 2, WS_REV = 4, WS_KDA = 8 };
// Bytes of the given parts, laid out one after another in the order FWD, KEEP, REV.
size_t tc_ws_bytes(const Geo &g, int parts);
// Sets the pointers of the given parts, carved from base in that order; leaves the others.
void tc_ws_carve(const Geo &g, int parts, void *base, TcWs *w);

// KDA's gate-scaled operands of every chunk (tc_prep.cu): w.Kt1 ... w.Kb, w.egc; with G
// (fp32 [chunks][64][dk], may be null) also the in-chunk cumulative log gate itself.
cudaError_t tc_kda_gates(const Geo &g, const Tensors &t, const TcWs &w, float *G, cudaStream_t s, Rec &rec);
// fp32 copies of the forward's chunk products and states (W, U~, P, S_n, U) for the CUDA-core
// backward kernels (tc_prep.cu).
cudaError_t tc_to_simt(const Geo &g, const TcWs &w, float *W, float *Ut, float *P, float *Sn, float *Un, cudaStream_t s,
                       Rec &rec);
// fp32 copies of the reverse chain's dS_{n+1} and dL/dU (tc_prep.cu).
cudaError_t tc_rev_to_simt(const Geo &g, const TcWs &w, float *dSn, float *dUn, cudaStream_t s, Rec &rec);
// The KDA backward's products with the chunk states on tcgen05, from the bf16 workspace tiles
// (S_n, dS_{n+1}, U, dU) and dO: Qd = dO S^T, dWm = -dU S^T, Tm = U dS+^T, RS = rowsum(S .* dS+),
// written to the CUDA-core workspace ([ci][C][dk] fp32 each; RS [ci][dk]).
cudaError_t tc_state_to_simt(const Geo &g, const Tensors &t, const TcWs &w, float *Qd, float *dWm, float *Tm,
                             float *RS, cudaStream_t s, Rec &rec);
// Per-chunk products (tc_prep.cu): g and beta, W, U~, P; with keep also T and k k^T.
// For KDA (no keep) from the operands of tc_kda_gates.
cudaError_t tc_chunk_prep(const Geo &g, const Tensors &t, const TcWs &w, bool keep, cudaStream_t s, Rec &rec);
// Forward state chain (tc_chain.cu).  mode 0: o, u, S_T; mode 1 (recompute for the
// backward): S_n and U of every chunk; mode 2: both.
cudaError_t tc_chain_fwd(const Geo &g, const Tensors &t, const TcWs &w, int mode, cudaStream_t s, Rec &rec);
// Reverse state chain (tc_chain.cu): dS_{n+1} and dL/dU of every chunk (w.dSn, w.dUn), the
// row sums w.skt, and dS0.  KDA reads the forward's gate-scaled q and k from w.
cudaError_t tc_chain_rev(const Geo &g, const Tensors &t, const TcWs &w, cudaStream_t s, Rec &rec);
// All intra-chunk gradients (tc_bwd.cu): dq, dk, dv, dbeta, d log alpha.
cudaError_t tc_bwd_chunk(const Geo &g, const Tensors &t, const TcWs &w, cudaStream_t s, Rec &rec);

}  // namespace dr
