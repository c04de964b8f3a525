/*
 * delta_rule.h -- C ABI of the B200 (sm_100a) chunkwise gated delta-rule library
 * (libdeltarule.so, built from gated_delta_rule_107_b200/csrc).
 *
 * The operation.  For every batch b and head h, with a state S in R^{dk x dv}
 * (row c = key channel), the library evaluates the recurrence of
 * "线性注意力架构演进与Kimi Delta Attention创新实践" (Kimi Delta Attention page),
 * section 2.1:
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 *
 * for three variants ("线性注意力架构：机制、权衡与跨层路由" explainer, core
 * method 1; ETH news article, section 二):
 *     DR_DELTANET  alpha_t == 1                      (no gate input)
 *     DR_GATED     one scalar alpha_t per token, head (Gated DeltaNet)
 *     DR_KDA       alpha_t in (0,1)^dk per channel    (Kimi Delta Attention)
 * and also returns the per-token write value that Cross-Layer Value Routing
 * forwards to the next layer (explainer section 4; chatpaper abstract):
 *     u_t = beta_t (v_t - (Diag(alpha_t) S_{t-1})^T k_t),
 * so that S_t = Diag(alpha_t) S_{t-1} + k_t u_t^T.
 *
 * It is computed chunk by chunk (chunks of `chunk` tokens, page section 6.1)
 * with the UT / WY transform of each chunk's triangular system (section 6.2)
 * and in-chunk cumulative gates accumulated in log space (section 7.1); the
 * state is carried in fp32 (section 7.2).  The result does not depend on the
 * chunk size except through rounding.
 *
 * Conventions shared by every entry point
 *   Layout     token-major, contiguous, row-major:
 *                q, k, dq, dk             [B, T, H, dk]
 *                v, out, u, dout, du, dv  [B, T, H, dv]
 *                alpha, dalpha            [B, T, H] (DR_GATED) or [B, T, H, dk] (DR_KDA);
 *                                         unused for DR_DELTANET (may be NULL)
 *                beta, dbeta              [B, T, H]
 *                S0, S_T, dS_T, dS0       [B, H, dk, dv], always fp32
 *   alpha      is the LOG gate, log(alpha_t) <= 0 (any real value is accepted;
 *              positive values grow the state).
 *   dtype      DR_F32 or DR_BF16: the element type of every per-token tensor
 *              (q, k, v, alpha, beta, out, u and all their gradients).  States are
 *              fp32.  Arithmetic is fp32 with fp32 accumulation; bf16 results are
 *              rounded to nearest-even once, at the store.
 *   Shapes     B, H >= 0; T >= 0; dk, dv in {64, 128}; chunk in {16, 32, 64}.
 *              T need not be a multiple of chunk (the tail chunk is masked).
 *              T == 0 is valid: the forward copies S0 (or zeros) to S_T and the
 *              backward copies dS_T (or zeros) to dS0.
 *   Pointers   device pointers (cudaMalloc / torch CUDA memory).  Tensors with a
 *              channel dimension (q, k, v, out, u, the KDA gate and all their
 *              gradients) and the fp32 states must be 16-byte aligned; beta, dbeta
 *              and the Gated-DeltaNet gate need only their element alignment.
 *              The caller owns every buffer; the library allocates no device
 *              memory, keeps no pointer after returning and has no global state
 *              except the device error word below and, once a call has run in
 *              segments (see Stream), one CUDA stream per device.  Inputs are never written.  Outputs must
 *              not alias inputs or each other.
 *   Workspace  caller-provided device scratch of at least
 *              delta_rule_workspace_size(...) bytes, 256-byte aligned; its
 *              contents on entry do not matter.  Two calls that run at the same
 *              time need distinct workspaces.
 *   Stream     `stream` is a cudaStream_t (NULL = the legacy default stream).  A
 *              call's work follows the work enqueued on it before and precedes
 *              the work enqueued after; the call returns without synchronising.
 *              The tensor-core forward and backward of long sequences with few
 *              (b, h) pairs (at most one (b, h) per 4 SMs, at least 32 chunks)
 *              run in four segments of the chunk range: part of their kernels
 *              on the library's own non-blocking stream, ordered against
 *              `stream` by events, which the call joins back before returning.
 *   Errors     every entry point validates its arguments first and returns a
 *              negative DR_ERR_* code without launching anything when they are
 *              bad.  Launch failures return DR_ERR_CUDA.  Faults detected on the
 *              device (a bounded wait that ran out) set a device error word that
 *              delta_rule_sync_status() reports.  Nothing prints, throws or aborts.
 */
#ifndef DELTA_RULE_H
#define DELTA_RULE_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { DR_DELTANET = 0, DR_GATED = 1, DR_KDA = 2 } dr_variant;
typedef enum { DR_F32 = 0, DR_BF16 = 1 } dr_dtype;

enum {
    DR_OK = 0,
    DR_ERR_ARG = -1,         /* bad shape, enum value, or missing required pointer */
    DR_ERR_UNSUPPORTED = -2, /* well-formed but not implemented (e.g. dk = 96)      */
    DR_ERR_ALIGN = -3,       /* a pointer is not 16-byte (workspace: 256-byte) aligned */
    DR_ERR_WORKSPACE = -4,   /* workspace missing or smaller than required          */
    DR_ERR_CUDA = -5,        /* a CUDA runtime call or kernel launch failed         */
    DR_ERR_TIMEOUT = -6      /* a device-side bounded wait expired (see sync_status) */
};

/*
 * Bytes of workspace that delta_rule_fwd (for_bwd = 0), delta_rule_bwd
 * (for_bwd = 1), delta_rule_fwd_save (for_bwd = 2) or delta_rule_bwd_saved
 * (for_bwd = 3) needs for these arguments.  Returns 0 when no workspace is
 * needed, and (size_t)-1 when the arguments are invalid.
 */
size_t delta_rule_workspace_size(int B, int T, int H, int dk, int dv, int variant, int chunk, int dtype,
                                 int for_bwd);

/*
 * Forward.  Evaluates the recurrence above from the initial state S0
 * (NULL = zero) and writes
 *   out  o_t = S_t^T q_t                                   (required)
 *   u    the write values u_t                              (NULL = not written)
 *   S_T  the state after the last token, fp32              (NULL = not written)
 */
int delta_rule_fwd(const void *q, const void *k, const void *v, const void *alpha, const void *beta, const float *S0,
                   void *out, void *u, float *S_T, int B, int T, int H, int dk, int dv, int variant, int chunk,
                   int dtype, void *workspace, size_t ws_bytes, void *stream);

/*
 * Backward.  Gradients of L = <dout, o> + <du, u> + <dS_T, S_T> with respect to
 * every forward input, for the same forward arguments.  du and dS_T may be NULL
 * (treated as zero).  Outputs: dq, dk_, dv_, dbeta (required); dalpha (the
 * gradient of the LOG gate, same shape as alpha; required for DR_GATED / DR_KDA,
 * ignored for DR_DELTANET); dS0 (fp32, NULL = not written).  The forward states
 * are recomputed inside the call (no saved activations are needed).
 */
int delta_rule_bwd(const void *q, const void *k, const void *v, const void *alpha, const void *beta, const float *S0,
                   const void *dout, const void *du, const float *dS_T, void *dq, void *dk_, void *dv_, void *dalpha,
                   void *dbeta, float *dS0, int B, int T, int H, int dk, int dv, int variant, int chunk, int dtype,
                   void *workspace, size_t ws_bytes, void *stream);

/*
 * Saved activations: a forward / backward pair for training.
 *
 * delta_rule_fwd_save computes exactly what delta_rule_fwd computes and, in
 * addition, keeps in the caller's buffer `saved` what the backward would
 * otherwise recompute: the per-chunk products of the chunked form (the
 * in-chunk cumulative log gate and beta, W, U~, P, T = (I + A)^-1, k k^T) and
 * the state entering every chunk with its write values, bf16 except the gate
 * (KDA: W, U~, P, the gate-scaled q e^g and k e^{g_C - g}, e^{g_C}, the states
 * and write values, and the per-channel cumulative log gate in fp32).
 * delta_rule_bwd_saved computes exactly what delta_rule_bwd computes for the
 * same forward arguments, reading `saved` instead of recomputing the forward.
 * `saved` must come from delta_rule_fwd_save on the same inputs and arguments
 * and must not change in between; the backward only reads it.
 *   delta_rule_saved_size  bytes of `saved` for these arguments (the buffer is
 *              device memory, 256-byte aligned).  It is 0 for configurations
 *              without a saved form: the saved form exists for all three
 *              variants with bf16 I/O, dk = dv = 128 and chunk 64.  For the
 *              others delta_rule_fwd_save behaves as delta_rule_fwd and
 *              delta_rule_bwd_saved as delta_rule_bwd, and `saved` may be NULL.
 *              Returns (size_t)-1 for invalid arguments.
 *   Workspace  delta_rule_workspace_size(..., for_bwd = 2) for the saving
 *              forward and (..., for_bwd = 3) for the backward from `saved`.
 *   Errors     DR_ERR_WORKSPACE when `saved` is needed and missing or smaller
 *              than delta_rule_saved_size; DR_ERR_ALIGN when it is not 256-byte
 *              aligned; otherwise as delta_rule_fwd / delta_rule_bwd.
 */
size_t delta_rule_saved_size(int B, int T, int H, int dk, int dv, int variant, int chunk, int dtype);
int delta_rule_fwd_save(const void *q, const void *k, const void *v, const void *alpha, const void *beta,
                        const float *S0, void *out, void *u, float *S_T, int B, int T, int H, int dk, int dv,
                        int variant, int chunk, int dtype, void *saved, size_t saved_bytes, void *workspace,
                        size_t ws_bytes, void *stream);
int delta_rule_bwd_saved(const void *q, const void *k, const void *v, const void *alpha, const void *beta,
                         const float *S0, const void *dout, const void *du, const float *dS_T, void *dq, void *dk_,
                         void *dv_, void *dalpha, void *dbeta, float *dS0, int B, int T, int H, int dk, int dv,
                         int variant, int chunk, int dtype, const void *saved, size_t saved_bytes, void *workspace,
                         size_t ws_bytes, void *stream);

/*
 * Measurement hooks.  delta_rule_launches() returns how many kernels one call
 * with these arguments launches -- delta_rule_fwd (for_bwd = 0), delta_rule_bwd
 * (1), delta_rule_fwd_save (2), delta_rule_bwd_saved (3) -- and stores a static
 * name for launch i in names[i] for i < max_names (names may be NULL); it
 * returns a negative DR_ERR_* code for invalid arguments.  The *_timed variants
 * compute what their plain entry points compute, bit for bit, but always with
 * one launch per kernel over the whole chunk range (never in segments; those
 * launches are what delta_rule_launches counts), and in addition record the
 * caller's cudaEvent_t events[i] (created handles) on `stream` immediately
 * before launch i and events[n] after the last launch (n = the launch count),
 * so that each kernel's device time is the elapsed time between consecutive
 * events.  n_events must be 0 (record nothing) or at least n + 1, else
 * DR_ERR_ARG.
 */
int delta_rule_launches(int B, int T, int H, int dk, int dv, int variant, int chunk, int dtype, int for_bwd,
                        const char **names, int max_names);
/* The number of kernels the plain entry point launches for these arguments (for_bwd as
 * above): delta_rule_launches' count, or more when the call runs in segments (see
 * Stream); a negative DR_ERR_* code for invalid arguments. */
int delta_rule_plain_launches(int B, int T, int H, int dk, int dv, int variant, int chunk, int dtype, int for_bwd);
int delta_rule_fwd_timed(const void *q, const void *k, const void *v, const void *alpha, const void *beta,
                         const float *S0, void *out, void *u, float *S_T, int B, int T, int H, int dk, int dv,
                         int variant, int chunk, int dtype, void *workspace, size_t ws_bytes, void *stream,
                         void *const *events, int n_events);
int delta_rule_bwd_timed(const void *q, const void *k, const void *v, const void *alpha, const void *beta,
                         const float *S0, const void *dout, const void *du, const float *dS_T, void *dq, void *dk_,
                         void *dv_, void *dalpha, void *dbeta, float *dS0, int B, int T, int H, int dk, int dv,
                         int variant, int chunk, int dtype, void *workspace, size_t ws_bytes, void *stream,
                         void *const *events, int n_events);
int delta_rule_fwd_save_timed(const void *q, const void *k, const void *v, const void *alpha, const void *beta,
                              const float *S0, void *out, void *u, float *S_T, int B, int T, int H, int dk, int dv,
                              int variant, int chunk, int dtype, void *saved, size_t saved_bytes, void *workspace,
                              size_t ws_bytes, void *stream, void *const *events, int n_events);
int delta_rule_bwd_saved_timed(const void *q, const void *k, const void *v, const void *alpha, const void *beta,
                               const float *S0, const void *dout, const void *du, const float *dS_T, void *dq,
                               void *dk_, void *dv_, void *dalpha, void *dbeta, float *dS0, int B, int T, int H,
                               int dk, int dv, int variant, int chunk, int dtype, const void *saved,
                               size_t saved_bytes, void *workspace, size_t ws_bytes, void *stream,
                               void *const *events, int n_events);

/*
 * Forward without any device allocation (no counterpart in the method; it is a
 * deployment convenience).  Some callers cannot call cudaMalloc at all: code
 * inside a CUDA graph being captured, allocator-less embedded runtimes, and
 * plugins that a host framework hands only their input and output buffers.
 * This entry point computes the same quantities as delta_rule_fwd (same
 * arguments, minus the workspace), always on the CUDA-core forward kernels,
 * with their scratch taken from a buffer of DELTA_RULE_NOALLOC_SCRATCH_BYTES
 * that is compiled into the library; every GPU that loads the library holds it
 * until the process exits.  The caller still passes every input and output.
 * Where delta_rule_fwd runs the same CUDA-core kernels (fp32 I/O, or dk = 64)
 * the results are bit-identical; where it takes the tensor-core path (bf16,
 * dk = 128) the two agree within the bf16 tolerance.
 *   - Problems whose scratch (delta_rule_workspace_size of the CUDA-core
 *     forward) exceeds the buffer return DR_ERR_WORKSPACE without launching;
 *     about 210 KB per (batch, head, chunk) at dk = dv = 128, chunk 64.
 *   - The first call on each device looks up the buffer's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.  The address is kept for the process: after
 *     cudaDeviceReset on a device it is stale, so do not call this entry point
 *     on that device again in the same process.
 *   - All calls on a device share the one buffer and it keeps the last call's
 *     contents (nothing in it needs to start at zero): calls whose kernels
 *     overlap on the GPU (different streams, or different threads without
 *     ordering) race and corrupt each other's results.
 */
#define DELTA_RULE_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
int delta_rule_fwd_noalloc(const void *q, const void *k, const void *v, const void *alpha, const void *beta,
                           const float *S0, void *out, void *u, float *S_T, int B, int T, int H, int dk, int dv,
                           int variant, int chunk, int dtype, void *stream);

/*
 * Fused forward: the pre-operation, the forward and the post-operation below in
 * the core's own kernels, with no pass over memory of their own (Kimi Delta
 * Attention page: section 7.1 -- q, k L2-normalised, logistic gates in log
 * space; section 4.1 -- sigmoid output gate on RMSNorm of the core's output).
 * From the raw projections q_raw, k_raw [B,T,H,dk], the raw forget logits
 * gate_raw [B,T,H] (Gated DeltaNet; unused and may be NULL for DeltaNet) and
 * the raw write-strength logits beta_raw [B,T,H] it computes what
 * delta_rule_preop then delta_rule_fwd then delta_rule_postop compute, to
 * within bf16 rounding (the normalised q, k and the gates stay in fp32 on chip;
 * sigmoid(gate_out) is formed in packed bf16 arithmetic with the hardware tanh,
 * and o enters y through a bf16 copy; y is within 1 % of the fp64 definition),
 *     y = RMSNorm(o) * w_norm * sigmoid(gate_out)   [B,T,H,dv]
 * and, when their pointers are not NULL, o itself (before the normalisation),
 * u and S_T.  gate_out [B,T,H,dv] has the I/O dtype, w_norm is fp32 [dv].
 * Served for Gated DeltaNet and DeltaNet with bf16 I/O, dk = dv = 128 and
 * chunk 64 (DR_ERR_UNSUPPORTED otherwise; the separate calls serve every
 * configuration).  The workspace is delta_rule_fwd_fused_workspace_size()
 * bytes ((size_t)-1 for arguments it does not serve), 256-byte aligned.
 * Errors, alignment and the asynchronous contract as delta_rule_fwd.
 */
size_t delta_rule_fwd_fused_workspace_size(int B, int T, int H, int dk, int dv, int variant, int chunk, int dtype);
int delta_rule_fwd_fused(const void *q_raw, const void *k_raw, const void *v, const void *gate_raw,
                         const void *beta_raw, const float *S0, const void *gate_out, const float *w_norm, void *y,
                         void *o, void *u, float *S_T, int B, int T, int H, int dk, int dv, int variant, int chunk,
                         int dtype, void *workspace, size_t ws_bytes, void *stream);

/*
 * Recurrent form for decoding.  Steps the recurrence above token by token from
 * the state S_in (NULL = zero) through the T tokens given and writes out and u
 * exactly as delta_rule_fwd does (u may be NULL), and the state after the last
 * token to S_out (NULL = not written).  S_out may be the same buffer as S_in
 * (the state is updated in place); partial overlap is not allowed.  It is meant
 * for the few tokens of a decoding step: each (b, h) keeps its state in
 * registers and reads and writes it once, with no chunking, workspace or saved
 * form.  For T == 0 it copies S_in (or zeros) to S_out.  Arguments, layouts,
 * alignment and errors follow the conventions above (no chunk argument).
 */
int delta_rule_decode(const void *q, const void *k, const void *v, const void *alpha, const void *beta,
                      const float *S_in, float *S_out, void *out, void *u, int B, int T, int H, int dk, int dv,
                      int variant, int dtype, void *stream);

/*
 * Pre- and post-operations around the core, one pass over memory each
 * (Kimi Delta Attention page: section 7.1 -- q, k L2-normalised after their
 * projections, a logistic forget gate biased to start near sigmoid(-3), decay
 * in log space; section 4.1 -- a sigmoid output gate on RMSNorm of the core's
 * output).  eps = 1e-6.  Rows are the B*T*H (token, head) pairs, token-major as
 * above; d = dk (pre) or dv (post) in {64, 128}; dtype as above for every
 * per-token tensor; the weight w and its gradient are fp32 [dv].
 *
 * delta_rule_preop: from the raw projections q_raw, k_raw [B,T,H,dk], the raw
 * write-strength logits beta_raw [B,T,H] and the raw forget logits gate_raw
 * ([B,T,H] Gated DeltaNet, [B,T,H,dk] KDA, unused and may be NULL for
 * DeltaNet), writes the core's inputs:
 *     q = q_raw / sqrt(|q_raw|^2 + eps),  k likewise        (per row)
 *     beta = sigmoid(beta_raw),  loga = -softplus(gate_raw)  (= log alpha)
 * delta_rule_preop_bwd: the gradients of <dq, q> + <dk_, k> + <dbeta, beta> +
 * <dloga, loga> with respect to q_raw, k_raw, beta_raw, gate_raw.
 *
 * delta_rule_postop: y = o / sqrt(mean(o^2) + eps) * w * sigmoid(gate) per row
 * of dv channels, for the core's output o, caller-computed gate logits gate
 * [B,T,H,dv] and the per-channel weight w (NULL = all ones).
 * delta_rule_postop_bwd: for dy [B,T,H,dv], the gradients do, dgate (required)
 * and dweight = the sum over all rows (NULL = not written).  It needs a
 * workspace of delta_rule_postop_workspace_size(dv) bytes (256-byte aligned);
 * dweight is summed in a fixed order, so results are deterministic.
 *
 * Outputs must not alias inputs.  Errors as for the other entry points.
 */
int delta_rule_preop(const void *q_raw, const void *k_raw, const void *beta_raw, const void *gate_raw, void *q,
                     void *k, void *beta, void *loga, int B, int T, int H, int dk, int variant, int dtype,
                     void *stream);
int delta_rule_preop_bwd(const void *q_raw, const void *k_raw, const void *beta_raw, const void *gate_raw,
                         const void *dq, const void *dk_, const void *dbeta, const void *dloga, void *dq_raw,
                         void *dk_raw, void *dbeta_raw, void *dgate_raw, int B, int T, int H, int dk, int variant,
                         int dtype, void *stream);
size_t delta_rule_postop_workspace_size(int dv);
int delta_rule_postop(const void *o, const void *gate, const float *weight, void *y, int B, int T, int H, int dv,
                      int dtype, void *stream);
int delta_rule_postop_bwd(const void *o, const void *gate, const float *weight, const void *dy, void *do_,
                          void *dgate, float *dweight, int B, int T, int H, int dv, int dtype, void *workspace,
                          size_t ws_bytes, void *stream);

/*
 * Short convolution (Kimi Delta Attention page, section 4.2: a depthwise
 * convolution of kernel size 4 on the q/k/v path).  Each of the D channels of a
 * token-major stream x [B,T,D] (for q, k or v: D = H*d, the [B,T,H,d] layout
 * above) is filtered causally with its own four taps w [D][4] (fp32, tap 3 on
 * the current token), across each sequence b separately:
 *     y[b,t,c] = sum_{j=0..3} w[c][j] * x[b, t-3+j, c]
 * where x at t < 0 is read from the three-token cache x_prev [B,3,D] (row 3+t;
 * NULL = zeros).  No bias and no activation.  cache_out [B,3,D] (NULL = not
 * written) receives the last three tokens of [x_prev ; x], which a later call on
 * the continuation of the stream takes as its x_prev; it must not alias x_prev.
 * D must be a multiple of 8 (else DR_ERR_UNSUPPORTED); x, x_prev, y, cache_out,
 * dy, dx, dx_prev 16-byte aligned; T = 0 writes only cache_out.
 *
 * delta_rule_shortconv_bwd: for dy [B,T,D], dx [B,T,D] (required when T > 0),
 * dw [D][4] = sum over b, t of dy[b,t,c] * x[b,t-3+j,c] (NULL = not written) and
 * dx_prev [B,3,D], the gradient of the cache tokens (NULL = not written).  dw
 * needs a workspace of delta_rule_shortconv_workspace_size(B, T, D) bytes
 * (256-byte aligned) and is summed in a fixed order (deterministic).  The
 * cache_out of the forward is a copy of input tokens; gradients reaching it are
 * the caller's to add to dx.
 */
size_t delta_rule_shortconv_workspace_size(int B, int T, int D);
int delta_rule_shortconv(const void *x, const float *w, const void *x_prev, void *y, void *cache_out, int B, int T,
                         int D, int dtype, void *stream);
int delta_rule_shortconv_bwd(const void *x, const float *w, const void *x_prev, const void *dy, void *dx, float *dw,
                             void *dx_prev, int B, int T, int D, int dtype, void *workspace, size_t ws_bytes,
                             void *stream);

/*
 * Cross-layer value routing (ETH news page on the architecture study, section 七;
 * the explainer's CLVR section): a layer's write values u (the u output of the
 * forward, [B,T,H,dv] read as an M x K matrix, M = B*T, K = H*dv) enter a higher
 * layer's hidden stream h [M,N] through a projection W [K,N] that starts at zero:
 *     h_out = h + u W          (h NULL: h_out = u W; h_out may alias h)
 * delta_rule_clvr_bwd: for dh_out [M,N], du = dh_out W^T [M,K] (NULL = not
 * written) and dW = u^T dh_out [K,N], fp32 (NULL = not written); the gradient of
 * h is dh_out itself.  u, W, h, h_out, dh_out and du have the I/O dtype.  bf16
 * runs the library's tcgen05 GEMM (bf16 operands read in place, transposed or
 * not, fp32 accumulation in tensor memory, the residual added in the epilogue;
 * dW's reduction over the M tokens is split into slices whose fp32 partials are
 * added in a fixed order), fp32 I/O a CUDA-core GEMM in fp32.  The caller passes
 * a workspace of delta_rule_clvr_workspace_size() bytes (256-byte aligned) for
 * those partials.  K and N must be multiples of 8; every pointer 16-byte aligned.
 */
size_t delta_rule_clvr_workspace_size(void);
int delta_rule_clvr(const void *u, const void *W, const void *h, void *h_out, int M, int K, int N, int dtype,
                    void *workspace, size_t ws_bytes, void *stream);
int delta_rule_clvr_bwd(const void *u, const void *W, const void *dh_out, void *du, float *dW, int M, int K, int N,
                        int dtype, void *workspace, size_t ws_bytes, void *stream);

/*
 * Self-test of failure detection.  Launches one kernel on `stream` whose bounded
 * wait (the same wait every pipelined kernel uses) waits for a barrier phase that
 * nothing completes; after limit_us microseconds (1 .. 1,000,000) it gives up,
 * raises the device error word and returns, so that the next
 * delta_rule_sync_status() reports DR_ERR_TIMEOUT and the context stays usable.
 * Returns DR_ERR_ARG for a limit out of range.
 */
int delta_rule_selftest_timeout(unsigned limit_us, void *stream);

/* Static text for a DR_* code ("ok", "invalid argument", ...). */
const char *delta_rule_strerror(int code);

/*
 * Synchronises `stream`, then reads and clears the calling device's error word.
 * Returns DR_OK, DR_ERR_TIMEOUT if a kernel reported an expired wait since the
 * last call, or DR_ERR_CUDA if the synchronisation itself failed.
 */
int delta_rule_sync_status(void *stream);

#ifdef __cplusplus
}
#endif
#endif /* DELTA_RULE_H */
