// tc_path.cuh -- the tcgen05 tensor-core path (bf16 I/O, dk = 128, chunk 64).
//
// Gated DeltaNet and DeltaNet at dv = 128 run the split path: a per-chunk kernel over all
// chunks at once (tc_prep.cu), the serial state chains (tc_chain.cu) and, for the
// backward, the per-chunk gradient kernel (tc_bwd.cu); api.cu sequences them.  KDA at
// dv = 128 runs the split forward after its gate kernels; Gated DeltaNet and DeltaNet at
// dv = 64 run the single-kernel forward of tc_fwd.cu.
#pragma once
#include "dr_common.cuh"

namespace dr {

bool tc_fwd_supported(const Geo &g, bool bf16);
// the single-kernel forward (Gated DeltaNet / DeltaNet, bf16, dk = 128); no workspace
cudaError_t tc_fwd(const Geo &g, const Tensors &t, void *workspace, cudaStream_t s, Rec &rec);
// number of launches of tc_fwd and their names
int tc_fwd_launches(const Geo &g, const char **names, int max_names);

// Split path: Gated DeltaNet / DeltaNet, bf16, dk = dv = 128, C = 64, and chunk row
// indices that fit the 32-bit coordinates of a TMA load.
bool tc_split_supported(const Geo &g, bool bf16);
// The same shapes for KDA: the split forward (the backward stays on the CUDA-core path).
bool tc_split_kda_supported(const Geo &g, bool bf16);

// Workspace of the split path, chunk-major (ci = (b H + h) N + n), every matrix row-major:
// bf16 tiles that later kernels load with TMA, plus fp32 per-token factors.  Parts:
//   WS_FWD    the forward's chunk products (gb, W, Ut, P);
//   WS_KEEP   the chunk products only the scalar-gate gradient kernel reads (Tn, KK);
//   WS_STATE  the chunk states and write values of the forward chain (Sn, Un);
//   WS_REV    what the reverse chain hands the gradient kernels (dSn, dUn, skt);
//   WS_KDA    KDA's forward-only gate-scaled operands (Kt1, Qt1, Kh, Kt, Dx);
//   WS_KDAC   KDA's operands of both chains (Qt, Kb, egc) and the chunk flags kwide;
//   WS_KDAG   KDA's in-chunk cumulative log gate G (fp32, read by its gradient kernel).
// Gated DeltaNet / DeltaNet: the forward's workspace is WS_FWD; the recomputing backward's
// FWD | KEEP | STATE | REV; the saved activations of delta_rule_fwd_save are FWD | KEEP | STATE,
// and the backward from them needs WS_REV as workspace.  KDA: the forward's workspace is
// FWD | KDA | KDAC; the saved activations are FWD | STATE | KDAC | KDAG (the saving forward's
// workspace WS_KDA), and the backward from them needs WS_REV beside the CUDA-core workspace.
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
    // KDA forward (channel-wise gates, g = in-chunk cumulative log gate per key channel).  The
    // pair factor e^{g_r - g_i} is split at a reference token of row r's 16-token block,
    // b(r) = 16 floor(r / 16):  e^{g_r - g_b(r)} e^{g_b(r) - g_i}.  For i before the block both
    // factors are <= 1; inside the block the second is >= 1 (at most e^{the block's span}).
    __nv_bfloat16 *Kt1;  // [ci][C][dk]   k e^{g - g_b}            (rows of P1's A)
    __nv_bfloat16 *Qt1;  // [ci][C][dk]   q e^{g - g_b}            (rows of P1's A)
    __nv_bfloat16 *Kh;   // [ci][KDA_KH_ROWS][dk]  P1's B: four sections, section R (R = 0..3)
                         //               at row 8 R (R + 1), rows i = 0 .. 16 R + 15:
                         //               k_i e^{g_16R - g_i} (exponent clamped at 80)
    __nv_bfloat16 *Kt;   // [ci][C][dk]   k e^{g}                  (W = T diag(beta) Kt)
    __nv_bfloat16 *Qt;   // [ci][C][dk]   q e^{g}                  (o = Qt S + P U)
    __nv_bfloat16 *Kb;   // [ci][C][dk]   k e^{g_C - g}            (S+ = Diag(e^{g_C}) S + Kb^T U)
    float *egc;          // [ci][dk]      e^{g_C}
    int *kwide;          // [ci]          1: some channel's gate falls by more than KDA_DIAG_SPAN
                         //               inside a 16-token block (the in-block factors would
                         //               leave the range where the split is exact)
    float *Dx;           // [ci][2][C][16] for such chunks only: the exact in-block sums
                         //               sum_c k_rc k_ic e^{g_rc - g_ic} ([0]) and
                         //               sum_c q_rc k_ic e^{g_rc - g_ic} ([1]), i = b(r) + 0..15
    float *G;            // [ci][C][dk]   KDA: g itself (fp32)
    float *rn;           // [ci][2][C]    fused forward: 1 / |k_r|, 1 / |q_r| of the raw rows
    int m0, m1;          // prep (and KDA gates), chains and the tensor-core gradient kernels: only
                         // the chunks [m0, m1) of each sequence (m1 = 0: all)
};
// rows of the stacked KDA column operand (16 + 32 + 48 + 64), and the widest in-block fall of
// a channel's cumulative log gate (nats) for which the block-reference split is used as is
constexpr int KDA_KH_ROWS = 160;
constexpr float KDA_DIAG_SPAN = 64.f;
enum { WS_FWD = 1, WS_KEEP = 2, WS_REV = 4, WS_KDA = 8, WS_STATE = 16, WS_KDAC = 32, WS_KDAG = 64, WS_RN = 128 };
// Bytes of the given parts, laid out one after another in the order FWD, KEEP, STATE, REV, KDA,
// KDAC, KDAG, RN (the row norms of the fused forward).
size_t tc_ws_bytes(const Geo &g, int parts);
// Sets the pointers of the given parts, carved from base in that order; leaves the others.
void tc_ws_carve(const Geo &g, int parts, void *base, TcWs *w);

// KDA's gate-scaled operands of every chunk (tc_prep.cu): w.Kt1 ... w.Kb, w.egc, w.kwide; with G
// (fp32 [chunks][64][dk], may be null) also the in-chunk cumulative log gate itself.  Then, for
// the chunks marked in w.kwide, the exact in-block sums w.Dx (a second kernel; the others exit).
cudaError_t tc_kda_gates(const Geo &g, const Tensors &t, const TcWs &w, float *G, cudaStream_t s, Rec &rec);
// fp32 copies of the forward's chunk products and states (W, U~, P, S_n, U) for the CUDA-core
// backward kernels (tc_prep.cu); with only (per-chunk flags), of the flagged chunks alone.
cudaError_t tc_to_simt(const Geo &g, const TcWs &w, float *W, float *Ut, float *P, float *Sn, float *Un, cudaStream_t s,
                       Rec &rec, const int *only = nullptr);
// fp32 copies of the reverse chain's dS_{n+1} and dL/dU (tc_prep.cu), likewise.
cudaError_t tc_rev_to_simt(const Geo &g, const TcWs &w, float *dSn, float *dUn, cudaStream_t s, Rec &rec,
                           const int *only = nullptr);
// The KDA backward's products with the chunk states on tcgen05, from the bf16 workspace tiles
// (S_n, dS_{n+1}, U, dU) and dO: Qd = dO S^T, dWm = -dU S^T, Tm = U dS+^T, RS = rowsum(S .* dS+),
// written to the CUDA-core workspace ([ci][C][dk] fp32 each; RS [ci][dk]).
cudaError_t tc_state_to_simt(const Geo &g, const Tensors &t, const TcWs &w, float *Qd, float *dWm, float *Tm,
                             float *RS, cudaStream_t s, Rec &rec, const int *only = nullptr);
// Per-chunk products (tc_prep.cu): g and beta, W, U~, P; with keep also T and k k^T.
// For KDA (no keep) from the operands of tc_kda_gates.  raw (Gated DeltaNet / DeltaNet, no
// keep): t.q, t.k are the raw projections and t.alpha, t.beta the raw logits; the prep applies
// the pre-operation (L2 normalisation, log alpha = -softplus, beta = sigmoid) on the fly and
// writes the row norms to w.rn.
cudaError_t tc_chunk_prep(const Geo &g, const Tensors &t, const TcWs &w, bool keep, cudaStream_t s, Rec &rec,
                          bool raw = false);
// Forward state chain (tc_chain.cu).  mode 0: o, u, S_T; mode 1 (recompute for the
// backward): S_n and U of every chunk; mode 2: both; mode 3 (Gated DeltaNet / DeltaNet): the
// fused forward of delta_rule_fwd_fused -- raw q, k with the row norms of w.rn, and the
// post-operation y = RMSNorm(o) w * sigmoid(gate) in the output epilogue (the two CTAs of a
// (b, h) form a cluster and exchange their halves' row sums of squares); o optional.
cudaError_t tc_chain_fwd(const Geo &g, const Tensors &t, const TcWs &w, int mode, cudaStream_t s, Rec &rec);
// Reverse state chain (tc_chain.cu): dS_{n+1} and dL/dU of every chunk (w.dSn, w.dUn), the
// row sums w.skt, and dS0.  KDA reads the forward's gate-scaled q and k from w.
cudaError_t tc_chain_rev(const Geo &g, const Tensors &t, const TcWs &w, cudaStream_t s, Rec &rec);
// All intra-chunk gradients (tc_bwd.cu): dq, dk, dv, dbeta, d log alpha.
cudaError_t tc_bwd_chunk(const Geo &g, const Tensors &t, const TcWs &w, cudaStream_t s, Rec &rec);
// KDA's intra-chunk gradients on tcgen05 (tc_bwd_kda.cu) for the chunks with w.kwide == 0, from the
// forward's W, U~, T, M (w.KK), states and write values and the reverse chain's dS_{n+1}, dU.
cudaError_t tc_bwd_kda(const Geo &g, const Tensors &t, const TcWs &w, cudaStream_t s, Rec &rec);

}  // namespace dr
