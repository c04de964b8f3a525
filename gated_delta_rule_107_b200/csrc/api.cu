// api.cu -- the C ABI declared in include/delta_rule.h.
//
// Argument validation, workspace planning and dispatch.  No compute happens on
// the host: every step of the path runs in the kernels of simt_path.cu and
// the tensor-core files and decode.cu.  Validation failures return before anything is enqueued.
#include <limits.h>

#include <mutex>

#include "../../include/delta_rule.h"
#include "decode.cuh"
#include "prepost.cuh"
#include "shortconv.cuh"
#include "clvr.cuh"
#include "dr_common.cuh"
#include "simt_path.cuh"
#include "tc_path.cuh"
#include "tc_ptx.cuh"

using namespace dr;

namespace dr {

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }
bool aligned_elem(const void *p, int dtype) { return ((uintptr_t)p & (dtype == DR_BF16 ? 1u : 3u)) == 0; }

// Checks shape / enum arguments; fills geo.  Returns DR_OK or an error code.
int check_shape(int B, int T, int H, int dk, int dv, int variant, int chunk, int dtype, Geo *geo) {
    if (B < 0 || T < 0 || H < 0) return DR_ERR_ARG;
    if (variant < DR_DELTANET || variant > DR_KDA) return DR_ERR_ARG;
    if (dtype != DR_F32 && dtype != DR_BF16) return DR_ERR_ARG;
    if (chunk != 16 && chunk != 32 && chunk != 64) return chunk > 0 ? DR_ERR_UNSUPPORTED : DR_ERR_ARG;
    if (dk <= 0 || dv <= 0) return DR_ERR_ARG;
    if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return DR_ERR_UNSUPPORTED;
    // every element index must fit comfortably in 63 bits; grids in 2^31 - 1 / 65535
    const double elems = (double)B * T * H * (dk > dv ? dk : dv);
    if (elems > 9.0e18 / 16) return DR_ERR_ARG;
    const long long N = T == 0 ? 0 : ((long long)T + chunk - 1) / chunk;
    if (N > INT_MAX || H > 65535 || B > 65535) return DR_ERR_UNSUPPORTED;
    geo->B = B; geo->T = T; geo->H = H; geo->dk = dk; geo->dv = dv; geo->C = chunk; geo->N = (int)N;
    geo->variant = variant;
    return DR_OK;
}

// Which kernels serve a call: the tensor-core forward for bf16, d = 128, C = 64.
bool use_tc_fwd(const Geo &g, int dtype) { return tc_fwd_supported(g, dtype == DR_BF16); }

// Call kinds: which entry point a size / plan question is about.
enum { K_FWD = 0, K_BWD = 1, K_FWD_SAVE = 2, K_BWD_SAVED = 3 };
bool is_bwd(int kind) { return kind == K_BWD || kind == K_BWD_SAVED; }

bool use_split(const Geo &g, int dtype) { return tc_split_supported(g, dtype == DR_BF16); }
// KDA's forward on the split path
bool use_split_kda(const Geo &g, int dtype, int kind) {
    return !is_bwd(kind) && tc_split_kda_supported(g, dtype == DR_BF16);
}
// KDA's backward: the forward's products and states and the reverse chain from the
// tensor-core kernels (widened to fp32), then the CUDA-core intra-chunk gradient kernels
bool use_kda_hybrid_bwd(const Geo &g, int dtype, int kind) {
    return is_bwd(kind) && tc_split_kda_supported(g, dtype == DR_BF16);
}
size_t ws_al(size_t x) { return (x + 255) & ~(size_t)255; }

// ---- segments of the chunk range (Gated DeltaNet / DeltaNet on the split path) ----
// The chain kernels run one CTA per (b, h, 64 value columns) and walk a sequence's chunks in
// order.  With few (b, h) pairs they occupy few SMs, so the chunk range is cut into segments: the
// prep of segment k + 1 runs on a second stream beside the forward chain of segment k, and the
// gradient kernel of segment k + 1 beside the reverse chain of segment k; the fp32 states at the
// cuts go through the workspace.  Each chain segment is enqueued before the kernel meant to run
// beside it, so that when both can start the chain's CTAs are placed first.
int seg_count(const Geo &g) {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 1;
    const long long chain_ctas = 2LL * g.B * g.H;  // (b, h, value half)
    if (chain_ctas * 2 > sms || g.N < 32) return 1;
    return 4;
}
size_t seg_cut_bytes(const Geo &g) {
    const int S = seg_count(g);
    return S > 1 ? ws_al((size_t)(S - 1) * g.B * g.H * g.dk * g.dv * sizeof(float)) : 0;
}
// the library's second stream on the current device (created once, non-blocking)
cudaStream_t side_stream() {
    static std::mutex mu;
    static cudaStream_t st[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!st[dev] && cudaStreamCreateWithFlags(&st[dev], cudaStreamNonBlocking) != cudaSuccess) st[dev] = nullptr;
    return st[dev];
}
struct SegEvents {  // events of one call, released when the call has enqueued its work
    cudaEvent_t ev[8] = {};
    int n = 0;
    bool make(int k) {
        for (n = 0; n < k; ++n)
            if (cudaEventCreateWithFlags(&ev[n], cudaEventDisableTiming) != cudaSuccess) return false;
        return true;
    }
    ~SegEvents() {
        for (int i = 0; i < n; ++i) cudaEventDestroy(ev[i]);
    }
};
int seg_bound(const Geo &g, int S, int k) { return (int)((long long)g.N * k / S); }

// prep (KDA: gates and prep; G as for tc_kda_gates) + forward chain in S segments; cuts: S - 1
// fp32 states [B, H, dk, dv]
cudaError_t fwd_segmented(const Geo &g, const Tensors &t, const TcWs &w, bool save, float *cuts, float *G,
                          cudaStream_t s) {
    const int S = seg_count(g);
    const size_t stride = (size_t)g.B * g.H * g.dk * g.dv;
    cudaStream_t ss = side_stream();
    SegEvents se;
    if (!ss || !se.make(S)) return cudaErrorMemoryAllocation;
    Rec none;
    const bool kda = g.variant == VAR_KDA;
    auto products = [&](const TcWs &ws, cudaStream_t st) -> cudaError_t {
        cudaError_t e2 = kda ? tc_kda_gates(g, t, ws, G, st, none) : cudaSuccess;
        return e2 == cudaSuccess ? tc_chunk_prep(g, t, ws, save, st, none) : e2;
    };
    TcWs wk = w;
    wk.m0 = seg_bound(g, S, 0); wk.m1 = seg_bound(g, S, 1);
    cudaError_t e = products(wk, s);
    if (e == cudaSuccess) e = cudaEventRecord(se.ev[0], s);
    for (int k = 0; k < S && e == cudaSuccess; ++k) {
        Tensors tk = t;
        tk.S0 = k == 0 ? t.S0 : cuts + (k - 1) * stride;
        tk.S_T = k == S - 1 ? t.S_T : cuts + k * stride;
        wk.m0 = seg_bound(g, S, k); wk.m1 = seg_bound(g, S, k + 1);
        if (k > 0) e = cudaStreamWaitEvent(s, se.ev[k], 0);
        if (e == cudaSuccess) e = tc_chain_fwd(g, tk, wk, save ? 2 : 0, s, none);
        if (e == cudaSuccess && k + 1 < S) {  // the next segment's products, beside this chain
            if (k == 0) e = cudaStreamWaitEvent(ss, se.ev[0], 0);
            wk.m0 = seg_bound(g, S, k + 1); wk.m1 = seg_bound(g, S, k + 2);
            if (e == cudaSuccess) e = products(wk, ss);
            if (e == cudaSuccess) e = cudaEventRecord(se.ev[k + 1], ss);
        }
    }
    return e;  // the last chain waited for the side stream's last prep
}

// reverse chain + gradient kernel (KDA: the tensor-core one) in S segments, the last segment
// first; cuts: S - 1 fp32 dL/dS
cudaError_t bwd_segmented(const Geo &g, const Tensors &t, const TcWs &w, float *cuts, cudaStream_t s) {
    const int S = seg_count(g);
    const size_t stride = (size_t)g.B * g.H * g.dk * g.dv;
    cudaStream_t ss = side_stream();
    SegEvents se;  // one per segment, and the side stream's end
    if (!ss || !se.make(S + 1)) return cudaErrorMemoryAllocation;
    Rec none;
    auto grads = [&](const TcWs &ws, cudaStream_t st) -> cudaError_t {
        return g.variant == VAR_KDA ? tc_bwd_kda(g, t, ws, st, none) : tc_bwd_chunk(g, t, ws, st, none);
    };
    TcWs wk = w;
    cudaError_t e = cudaSuccess;
    for (int k = S - 1; k >= 0 && e == cudaSuccess; --k) {
        Tensors tk = t;
        tk.dS_T = k == S - 1 ? t.dS_T : cuts + k * stride;  // dL/dS after the segment
        tk.dS0 = k == 0 ? t.dS0 : cuts + (k - 1) * stride;   // dL/dS entering it
        wk.m0 = seg_bound(g, S, k); wk.m1 = seg_bound(g, S, k + 1);
        e = tc_chain_rev(g, tk, wk, s, none);
        if (e == cudaSuccess) e = cudaEventRecord(se.ev[k], s);
        if (e == cudaSuccess && k + 1 < S) {  // the gradients of the segment after, beside this chain
            wk.m0 = seg_bound(g, S, k + 1); wk.m1 = seg_bound(g, S, k + 2);
            e = cudaStreamWaitEvent(ss, se.ev[k + 1], 0);
            if (e == cudaSuccess) e = grads(wk, ss);
        }
    }
    if (e == cudaSuccess) {  // the first segment's gradients on the caller's stream; then join
        wk.m0 = seg_bound(g, S, 0); wk.m1 = seg_bound(g, S, 1);
        e = grads(wk, s);
    }
    if (e == cudaSuccess) e = cudaEventRecord(se.ev[S], ss);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, se.ev[S], 0);
    return e;
}

// Parts of the split-path workspace (tc_path.cuh) that each call kind uses
constexpr int GDN_SAVED = WS_FWD | WS_KEEP | WS_STATE;
constexpr int KDA_FWD = WS_FWD | WS_KDA | WS_KDAC;
constexpr int KDA_SAVED = WS_FWD | WS_KEEP | WS_STATE | WS_KDAC | WS_KDAG;
constexpr int KDA_BWD = WS_FWD | WS_KEEP | WS_STATE | WS_REV | WS_KDA | WS_KDAC;

size_t ws_bytes(const Geo &g, int dtype, int kind) {
    if (g.T == 0 || g.B == 0 || g.H == 0) return 0;
    if (use_split(g, dtype)) {
        // the parts below, then (only for shapes cut into segments) the states at the cuts
        const size_t cut = seg_cut_bytes(g);
        auto with_cut = [&](size_t x) { return cut ? ws_al(x) + cut : x; };
        switch (kind) {
            case K_FWD: return with_cut(tc_ws_bytes(g, WS_FWD));
            case K_BWD: return with_cut(tc_ws_bytes(g, GDN_SAVED | WS_REV));
            case K_FWD_SAVE: return cut;  // everything it keeps lives in the saved buffer
            default: return with_cut(tc_ws_bytes(g, WS_REV));
        }
    }
    if (use_split_kda(g, dtype, kind)) {  // the saving forward keeps all but its forward-only tiles
        const size_t x = tc_ws_bytes(g, kind == K_FWD_SAVE ? WS_KDA : KDA_FWD), cut = seg_cut_bytes(g);
        return cut ? ws_al(x) + cut : x;  // (the states at the cuts of a segmented call after them)
    }
    if (use_kda_hybrid_bwd(g, dtype, kind)) {
        const size_t x = ws_al(simt_ws_bytes(g, true)) + tc_ws_bytes(g, kind == K_BWD_SAVED ? WS_REV : KDA_BWD),
                     cut = seg_cut_bytes(g);
        return cut ? ws_al(x) + cut : x;
    }
    if (!is_bwd(kind) && use_tc_fwd(g, dtype)) return 0;
    return simt_ws_bytes(g, is_bwd(kind));
}

// Bytes of the saved-activation buffer (0: no saved form for this configuration).
size_t saved_bytes(const Geo &g, int dtype) {
    if (g.T == 0 || g.B == 0 || g.H == 0) return 0;
    if (use_split(g, dtype)) return tc_ws_bytes(g, GDN_SAVED);
    if (tc_split_kda_supported(g, dtype == DR_BF16)) return tc_ws_bytes(g, KDA_SAVED);
    return 0;
}

// Checks a caller buffer of `given` bytes against `need` (256-byte aligned when needed).
int check_buffer(const void *p, size_t given, size_t need) {
    if (need == 0) return DR_OK;
    if (!p || given < need) return DR_ERR_WORKSPACE;
    if (((uintptr_t)p & 255u) != 0) return DR_ERR_ALIGN;
    return DR_OK;
}

int launch_status(cudaError_t e) { return e == cudaSuccess ? DR_OK : DR_ERR_CUDA; }

// T == 0: S_T := S0 (or 0), dS0 := dS_T (or 0).
int copy_state(float *dst, const float *src, const Geo &g, cudaStream_t s) {
    if (!dst) return DR_OK;
    const size_t bytes = (size_t)g.B * g.H * g.dk * g.dv * sizeof(float);
    if (bytes == 0) return DR_OK;
    cudaError_t e = src ? cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, s) : cudaMemsetAsync(dst, 0, bytes, s);
    return launch_status(e);
}

}  // namespace dr

extern "C" size_t delta_rule_workspace_size(int B, int T, int H, int dk, int dv, int variant, int chunk, int dtype,
                                            int for_bwd) {
    Geo g;
    if (check_shape(B, T, H, dk, dv, variant, chunk, dtype, &g) != DR_OK) return (size_t)-1;
    if (for_bwd < 0 || for_bwd > 3) return (size_t)-1;
    return ws_bytes(g, dtype, for_bwd);
}

extern "C" size_t delta_rule_saved_size(int B, int T, int H, int dk, int dv, int variant, int chunk, int dtype) {
    Geo g;
    if (check_shape(B, T, H, dk, dv, variant, chunk, dtype, &g) != DR_OK) return (size_t)-1;
    return saved_bytes(g, dtype);
}

// save: the saving forward (kind K_FWD_SAVE) with its buffer `saved`
static int fwd_impl(const void *q, const void *k, const void *v, const void *alpha, const void *beta,
                    const float *S0, void *out, void *u, float *S_T, int B, int T, int H, int dk, int dv, int variant,
                    int chunk, int dtype, bool save, void *saved, size_t saved_given, void *workspace,
                    size_t ws_bytes_given, void *stream, Rec &rec) {
    Geo g;
    int rc = check_shape(B, T, H, dk, dv, variant, chunk, dtype, &g);
    if (rc != DR_OK) return rc;
    cudaStream_t s = (cudaStream_t)stream;
    const bool empty = (size_t)B * H == 0;
    if (T == 0 || empty) return empty ? DR_OK : copy_state(S_T, S0, g, s);
    if (!q || !k || !v || !beta || !out) return DR_ERR_ARG;
    if (variant != DR_DELTANET && !alpha) return DR_ERR_ARG;
    // tiles moved by TMA / vector accesses need 16 B; per-token scalars only their element size
    const void *ptrs[] = {q, k, v, variant == DR_KDA ? alpha : nullptr, S0, out, u, S_T};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return DR_ERR_ALIGN;
    if (!aligned_elem(beta, dtype) || (variant == DR_GATED && !aligned_elem(alpha, dtype))) return DR_ERR_ALIGN;
    const int kind = save ? K_FWD_SAVE : K_FWD;
    rc = check_buffer(workspace, ws_bytes_given, ws_bytes(g, dtype, kind));
    if (rc == DR_OK && save) rc = check_buffer(saved, saved_given, saved_bytes(g, dtype));
    if (rc != DR_OK) return rc;
    Tensors t = {};
    t.q = q; t.k = k; t.v = v; t.alpha = alpha; t.beta = beta; t.S0 = S0; t.out = out; t.u = u; t.S_T = S_T;
    if (use_split(g, dtype)) {
        TcWs w = {};
        if (save) tc_ws_carve(g, GDN_SAVED, saved, &w);
        else tc_ws_carve(g, WS_FWD, workspace, &w);
        if (seg_count(g) > 1 && rec.ev == nullptr) {  // (the timed entry points run one launch each)
            float *cuts = (float *)((char *)workspace + (save ? 0 : ws_al(tc_ws_bytes(g, WS_FWD))));
            rc = launch_status(fwd_segmented(g, t, w, save, cuts, nullptr, s));
        } else {
            rc = launch_status(tc_chunk_prep(g, t, w, save, s, rec));
            if (rc == DR_OK) rc = launch_status(tc_chain_fwd(g, t, w, save ? 2 : 0, s, rec));
        }
    } else if (use_split_kda(g, dtype, kind)) {
        TcWs w = {};
        if (save) {  // the chain operands, states and G go to the saved buffer
            tc_ws_carve(g, KDA_SAVED, saved, &w);
            tc_ws_carve(g, WS_KDA, workspace, &w);
        } else {
            tc_ws_carve(g, KDA_FWD, workspace, &w);
        }
        if (seg_count(g) > 1 && rec.ev == nullptr) {
            float *cuts = (float *)((char *)workspace + ws_al(tc_ws_bytes(g, save ? WS_KDA : KDA_FWD)));
            rc = launch_status(fwd_segmented(g, t, w, save, cuts, save ? w.G : nullptr, s));
        } else {
            rc = launch_status(tc_kda_gates(g, t, w, save ? w.G : nullptr, s, rec));
            if (rc == DR_OK) rc = launch_status(tc_chunk_prep(g, t, w, save, s, rec));
            if (rc == DR_OK) rc = launch_status(tc_chain_fwd(g, t, w, save ? 2 : 0, s, rec));
        }
    } else if (use_tc_fwd(g, dtype)) {
        rc = launch_status(tc_fwd(g, t, workspace, s, rec));
    } else {
        const SimtWs w = simt_ws_carve(g, false, workspace);
        rc = launch_status(simt_fwd(g, t, dtype == DR_BF16, w, s, rec));
    }
    rec.mark(s);  // end of the last launch
    return rc;
}

// from_saved: the backward from saved activations (kind K_BWD_SAVED) with its buffer `saved`
static int bwd_impl(const void *q, const void *k, const void *v, const void *alpha, const void *beta,
                    const float *S0, const void *dout, const void *du, const float *dS_T, void *dq, void *dk_,
                    void *dv_, void *dalpha, void *dbeta, float *dS0, int B, int T, int H, int dk, int dv, int variant,
                    int chunk, int dtype, bool from_saved, const void *saved, size_t saved_given, void *workspace,
                    size_t ws_bytes_given, void *stream, Rec &rec) {
    Geo g;
    int rc = check_shape(B, T, H, dk, dv, variant, chunk, dtype, &g);
    if (rc != DR_OK) return rc;
    cudaStream_t s = (cudaStream_t)stream;
    const bool empty = (size_t)B * H == 0;
    if (T == 0 || empty) return empty ? DR_OK : copy_state(dS0, dS_T, g, s);
    if (!q || !k || !v || !beta || !dout || !dq || !dk_ || !dv_ || !dbeta) return DR_ERR_ARG;
    if (variant != DR_DELTANET && (!alpha || !dalpha)) return DR_ERR_ARG;
    const void *ptrs[] = {q, k, v, variant == DR_KDA ? alpha : nullptr, S0, dout, du, dS_T, dq, dk_, dv_,
                          variant == DR_KDA ? dalpha : nullptr, dS0};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return DR_ERR_ALIGN;
    if (!aligned_elem(beta, dtype) || !aligned_elem(dbeta, dtype)) return DR_ERR_ALIGN;
    if (variant == DR_GATED && (!aligned_elem(alpha, dtype) || !aligned_elem(dalpha, dtype))) return DR_ERR_ALIGN;
    const int kind = from_saved ? K_BWD_SAVED : K_BWD;
    rc = check_buffer(workspace, ws_bytes_given, ws_bytes(g, dtype, kind));
    if (rc == DR_OK && from_saved) rc = check_buffer(saved, saved_given, saved_bytes(g, dtype));
    if (rc != DR_OK) return rc;
    Tensors t = {};
    t.q = q; t.k = k; t.v = v; t.alpha = alpha; t.beta = beta; t.S0 = S0;
    t.dout = dout; t.du = du; t.dS_T = dS_T;
    t.dq = dq; t.dk = dk_; t.dv = dv_; t.dalpha = dalpha; t.dbeta = dbeta; t.dS0 = dS0;
    if (use_split(g, dtype)) {
        TcWs w = {};
        if (from_saved) {
            tc_ws_carve(g, GDN_SAVED, const_cast<void *>(saved), &w);
            tc_ws_carve(g, WS_REV, workspace, &w);
        } else {
            tc_ws_carve(g, GDN_SAVED | WS_REV, workspace, &w);
            rc = launch_status(tc_chunk_prep(g, t, w, true, s, rec));
            if (rc == DR_OK) rc = launch_status(tc_chain_fwd(g, t, w, 1, s, rec));
        }
        if (rc == DR_OK && seg_count(g) > 1 && rec.ev == nullptr) {
            float *cuts = (float *)((char *)workspace + ws_al(tc_ws_bytes(g, from_saved ? WS_REV : (GDN_SAVED | WS_REV))));
            rc = launch_status(bwd_segmented(g, t, w, cuts, s));
        } else {
            if (rc == DR_OK) rc = launch_status(tc_chain_rev(g, t, w, s, rec));
            if (rc == DR_OK) rc = launch_status(tc_bwd_chunk(g, t, w, s, rec));
        }
    } else if (use_kda_hybrid_bwd(g, dtype, kind)) {
        SimtWs sw = simt_ws_carve(g, true, workspace);
        char *tcbase = (char *)workspace + ws_al(simt_ws_bytes(g, true));
        TcWs w = {};
        if (from_saved) {  // the saving forward's chain operands, states and G
            tc_ws_carve(g, KDA_SAVED, const_cast<void *>(saved), &w);
            tc_ws_carve(g, WS_REV, tcbase, &w);
            sw.G = w.G;
        } else {
            tc_ws_carve(g, KDA_BWD, tcbase, &w);
            rc = launch_status(tc_kda_gates(g, t, w, sw.G, s, rec));
            if (rc == DR_OK) rc = launch_status(tc_chunk_prep(g, t, w, true, s, rec));
            if (rc == DR_OK) rc = launch_status(tc_chain_fwd(g, t, w, 1, s, rec));
        }
        // the intra-chunk gradients on tcgen05 for every chunk whose gates stay within the block
        // split's range; the others (w.kwide) on the CUDA-core kernel, which reads W, U~, U, dU
        // widened to fp32 and the state products (these kernels pass over the other chunks)
        if (rc == DR_OK && seg_count(g) > 1 && rec.ev == nullptr) {
            float *cuts = (float *)((char *)workspace + ws_al(ws_al(simt_ws_bytes(g, true)) +
                                                              tc_ws_bytes(g, from_saved ? WS_REV : KDA_BWD)));
            rc = launch_status(bwd_segmented(g, t, w, cuts, s));
        } else {
            if (rc == DR_OK) rc = launch_status(tc_chain_rev(g, t, w, s, rec));
            if (rc == DR_OK) rc = launch_status(tc_bwd_kda(g, t, w, s, rec));
        }
        sw.only = w.kwide;
        if (rc == DR_OK) rc = launch_status(tc_to_simt(g, w, sw.W, sw.Ut, nullptr, nullptr, sw.Un, s, rec, w.kwide));
        if (rc == DR_OK) rc = launch_status(tc_rev_to_simt(g, w, nullptr, sw.dUn, s, rec, w.kwide));
        if (rc == DR_OK)
            rc = launch_status(tc_state_to_simt(g, t, w, sw.Qd, sw.dWm, sw.Tm, sw.RS, s, rec, w.kwide));
        if (rc == DR_OK) rc = launch_status(simt_bwd_intra(g, t, dtype == DR_BF16, sw, s, rec));
    } else {
        const SimtWs w = simt_ws_carve(g, true, workspace);
        rc = launch_status(simt_bwd(g, t, dtype == DR_BF16, w, s, rec));
    }
    rec.mark(s);  // end of the last launch
    return rc;
}

// The fused forward: pre-operation, core forward and post-operation in the split path's two
// kernels (Gated DeltaNet / DeltaNet, bf16, dk = dv = 128, chunk 64).
static int fused_shape(int B, int T, int H, int dk, int dv, int variant, int chunk, int dtype, Geo *g) {
    const int rc = check_shape(B, T, H, dk, dv, variant, chunk, dtype, g);
    if (rc != DR_OK) return rc;
    return use_split(*g, dtype) ? DR_OK : DR_ERR_UNSUPPORTED;
}

extern "C" size_t delta_rule_fwd_fused_workspace_size(int B, int T, int H, int dk, int dv, int variant, int chunk,
                                                      int dtype) {
    Geo g;
    if (fused_shape(B, T, H, dk, dv, variant, chunk, dtype, &g) != DR_OK) return (size_t)-1;
    if (g.T == 0 || g.B == 0 || g.H == 0) return 0;
    return tc_ws_bytes(g, WS_FWD | WS_RN);
}

extern "C" int delta_rule_fwd_fused(const void *q_raw, const void *k_raw, const void *v, const void *gate_raw,
                                    const void *beta_raw, const float *S0, const void *gate_out, const float *w_norm,
                                    void *y, void *o, void *u, float *S_T, int B, int T, int H, int dk, int dv,
                                    int variant, int chunk, int dtype, void *workspace, size_t ws_bytes_given,
                                    void *stream) {
    Geo g;
    int rc = fused_shape(B, T, H, dk, dv, variant, chunk, dtype, &g);
    if (rc != DR_OK) return rc;
    cudaStream_t s = (cudaStream_t)stream;
    const bool empty = (size_t)B * H == 0;
    if (T == 0 || empty) return empty ? DR_OK : copy_state(S_T, S0, g, s);
    if (!q_raw || !k_raw || !v || !beta_raw || !gate_out || !w_norm || !y) return DR_ERR_ARG;
    if (variant != DR_DELTANET && !gate_raw) return DR_ERR_ARG;
    const void *ptrs[] = {q_raw, k_raw, v, S0, gate_out, w_norm, y, o, u, S_T};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return DR_ERR_ALIGN;
    if (!aligned_elem(beta_raw, dtype) || (variant == DR_GATED && !aligned_elem(gate_raw, dtype))) return DR_ERR_ALIGN;
    rc = check_buffer(workspace, ws_bytes_given, tc_ws_bytes(g, WS_FWD | WS_RN));
    if (rc != DR_OK) return rc;
    Tensors t = {};
    t.q = q_raw; t.k = k_raw; t.v = v; t.alpha = gate_raw; t.beta = beta_raw; t.S0 = S0;
    t.out = o; t.u = u; t.S_T = S_T; t.gate_o = gate_out; t.w_norm = w_norm; t.y = y;
    TcWs w = {};
    tc_ws_carve(g, WS_FWD | WS_RN, workspace, &w);
    Rec rec;
    rc = launch_status(tc_chunk_prep(g, t, w, false, s, rec, true));
    if (rc == DR_OK) rc = launch_status(tc_chain_fwd(g, t, w, 3, s, rec));
    return rc;
}

// Number of kernel launches of one call and their names (launch order).
static int launch_plan(const Geo &g, int dtype, int kind, const char **names, int max_names) {
    static const char *const SPLIT_FWD[2] = {"k_chunk_prep", "k_chain_fwd"};
    static const char *const SPLIT_FWD_SAVE[2] = {"k_chunk_prep(keep)", "k_chain_fwd(keep)"};
    static const char *const SPLIT_BWD[4] = {"k_chunk_prep(keep)", "k_chain_fwd(recompute)", "k_chain_rev",
                                             "k_bwd_chunk_tc"};
    static const char *const SPLIT_BWD_SAVED[2] = {"k_chain_rev", "k_bwd_chunk_tc"};
    static const char *const SPLIT_KDA_FWD[4] = {"k_kda_gates", "k_kda_diag", "k_chunk_prep", "k_chain_fwd"};
    static const char *const KDA_BWD_NAMES[10] = {"k_kda_gates", "k_kda_diag", "k_chunk_prep(keep)",
                                                  "k_chain_fwd(recompute)", "k_chain_rev", "k_bwd_kda_tc", "k_widen",
                                                  "k_widen", "k_state_tc", "k_bwd_intra"};
    static const char *const KDA_FWD_SAVE[4] = {"k_kda_gates", "k_kda_diag", "k_chunk_prep(keep)", "k_chain_fwd(keep)"};
    int n = 0;
    const char *const *src = nullptr;
    if (g.T == 0 || g.B == 0 || g.H == 0) return 0;
    if (use_split(g, dtype)) {
        switch (kind) {
            case K_FWD: src = SPLIT_FWD; n = 2; break;
            case K_FWD_SAVE: src = SPLIT_FWD_SAVE; n = 2; break;
            case K_BWD: src = SPLIT_BWD; n = 4; break;
            default: src = SPLIT_BWD_SAVED; n = 2; break;
        }
    } else if (use_split_kda(g, dtype, kind)) {
        src = kind == K_FWD_SAVE ? KDA_FWD_SAVE : SPLIT_KDA_FWD;
        n = 4;
    } else if (use_kda_hybrid_bwd(g, dtype, kind)) {
        src = kind == K_BWD_SAVED ? KDA_BWD_NAMES + 4 : KDA_BWD_NAMES;  // from saved: no recompute
        n = kind == K_BWD_SAVED ? 6 : 10;
    } else if (!is_bwd(kind) && use_tc_fwd(g, dtype)) {
        return tc_fwd_launches(g, names, max_names);
    } else {
        src = is_bwd(kind) ? SIMT_BWD_KERNELS : SIMT_FWD_KERNELS;
        n = is_bwd(kind) ? 5 : 3;
    }
    for (int i = 0; names && i < n && i < max_names; ++i) names[i] = src[i];
    return n;
}

static int make_rec(const Geo &g, int dtype, int kind, void *const *events, int n_events, Rec *rec) {
    if (n_events == 0 || events == nullptr) return DR_OK;
    const int n = launch_plan(g, dtype, kind, nullptr, 0);
    if (n_events < n + 1) return DR_ERR_ARG;
    rec->ev = (cudaEvent_t *)events;
    rec->n = n + 1;
    return DR_OK;
}

extern "C" int delta_rule_fwd(const void *q, const void *k, const void *v, const void *alpha, const void *beta,
                              const float *S0, void *out, void *u, float *S_T, int B, int T, int H, int dk, int dv,
                              int variant, int chunk, int dtype, void *workspace, size_t ws_bytes_given,
                              void *stream) {
    Rec rec;
    return fwd_impl(q, k, v, alpha, beta, S0, out, u, S_T, B, T, H, dk, dv, variant, chunk, dtype, false, nullptr, 0,
                    workspace, ws_bytes_given, stream, rec);
}

extern "C" int delta_rule_fwd_save(const void *q, const void *k, const void *v, const void *alpha, const void *beta,
                                   const float *S0, void *out, void *u, float *S_T, int B, int T, int H, int dk,
                                   int dv, int variant, int chunk, int dtype, void *saved, size_t saved_given,
                                   void *workspace, size_t ws_bytes_given, void *stream) {
    Rec rec;
    return fwd_impl(q, k, v, alpha, beta, S0, out, u, S_T, B, T, H, dk, dv, variant, chunk, dtype, true, saved,
                    saved_given, workspace, ws_bytes_given, stream, rec);
}

static int fwd_timed(const void *q, const void *k, const void *v, const void *alpha, const void *beta,
                     const float *S0, void *out, void *u, float *S_T, int B, int T, int H, int dk, int dv, int variant,
                     int chunk, int dtype, bool save, void *saved, size_t saved_given, void *workspace,
                     size_t ws_bytes_given, void *stream, void *const *events, int n_events) {
    Geo g;
    int rc = check_shape(B, T, H, dk, dv, variant, chunk, dtype, &g);
    if (rc != DR_OK) return rc;
    Rec rec;
    rc = make_rec(g, dtype, save ? K_FWD_SAVE : K_FWD, events, n_events, &rec);
    if (rc != DR_OK) return rc;
    rc = fwd_impl(q, k, v, alpha, beta, S0, out, u, S_T, B, T, H, dk, dv, variant, chunk, dtype, save, saved,
                  saved_given, workspace, ws_bytes_given, stream, rec);
    return (rc == DR_OK && rec.bad) ? DR_ERR_ARG : rc;
}

extern "C" int delta_rule_fwd_timed(const void *q, const void *k, const void *v, const void *alpha, const void *beta,
                                    const float *S0, void *out, void *u, float *S_T, int B, int T, int H, int dk,
                                    int dv, int variant, int chunk, int dtype, void *workspace, size_t ws_bytes_given,
                                    void *stream, void *const *events, int n_events) {
    return fwd_timed(q, k, v, alpha, beta, S0, out, u, S_T, B, T, H, dk, dv, variant, chunk, dtype, false, nullptr, 0,
                     workspace, ws_bytes_given, stream, events, n_events);
}

extern "C" int delta_rule_fwd_save_timed(const void *q, const void *k, const void *v, const void *alpha,
                                         const void *beta, const float *S0, void *out, void *u, float *S_T, int B,
                                         int T, int H, int dk, int dv, int variant, int chunk, int dtype, void *saved,
                                         size_t saved_given, void *workspace, size_t ws_bytes_given, void *stream,
                                         void *const *events, int n_events) {
    return fwd_timed(q, k, v, alpha, beta, S0, out, u, S_T, B, T, H, dk, dv, variant, chunk, dtype, true, saved,
                     saved_given, workspace, ws_bytes_given, stream, events, n_events);
}

extern "C" int delta_rule_bwd(const void *q, const void *k, const void *v, const void *alpha, const void *beta,
                              const float *S0, const void *dout, const void *du, const float *dS_T, void *dq,
                              void *dk_, void *dv_, void *dalpha, void *dbeta, float *dS0, int B, int T, int H, int dk,
                              int dv, int variant, int chunk, int dtype, void *workspace, size_t ws_bytes_given,
                              void *stream) {
    Rec rec;
    return bwd_impl(q, k, v, alpha, beta, S0, dout, du, dS_T, dq, dk_, dv_, dalpha, dbeta, dS0, B, T, H, dk, dv,
                    variant, chunk, dtype, false, nullptr, 0, workspace, ws_bytes_given, stream, rec);
}

extern "C" int delta_rule_bwd_saved(const void *q, const void *k, const void *v, const void *alpha, const void *beta,
                                    const float *S0, const void *dout, const void *du, const float *dS_T, void *dq,
                                    void *dk_, void *dv_, void *dalpha, void *dbeta, float *dS0, int B, int T, int H,
                                    int dk, int dv, int variant, int chunk, int dtype, const void *saved,
                                    size_t saved_given, void *workspace, size_t ws_bytes_given, void *stream) {
    Rec rec;
    return bwd_impl(q, k, v, alpha, beta, S0, dout, du, dS_T, dq, dk_, dv_, dalpha, dbeta, dS0, B, T, H, dk, dv,
                    variant, chunk, dtype, true, saved, saved_given, workspace, ws_bytes_given, stream, rec);
}

static int bwd_timed(const void *q, const void *k, const void *v, const void *alpha, const void *beta,
                     const float *S0, const void *dout, const void *du, const float *dS_T, void *dq, void *dk_,
                     void *dv_, void *dalpha, void *dbeta, float *dS0, int B, int T, int H, int dk, int dv,
                     int variant, int chunk, int dtype, bool from_saved, const void *saved, size_t saved_given,
                     void *workspace, size_t ws_bytes_given, void *stream, void *const *events, int n_events) {
    Geo g;
    int rc = check_shape(B, T, H, dk, dv, variant, chunk, dtype, &g);
    if (rc != DR_OK) return rc;
    Rec rec;
    rc = make_rec(g, dtype, from_saved ? K_BWD_SAVED : K_BWD, events, n_events, &rec);
    if (rc != DR_OK) return rc;
    rc = bwd_impl(q, k, v, alpha, beta, S0, dout, du, dS_T, dq, dk_, dv_, dalpha, dbeta, dS0, B, T, H, dk, dv,
                  variant, chunk, dtype, from_saved, saved, saved_given, workspace, ws_bytes_given, stream, rec);
    return (rc == DR_OK && rec.bad) ? DR_ERR_ARG : rc;
}

extern "C" int delta_rule_bwd_timed(const void *q, const void *k, const void *v, const void *alpha,
                                    const void *beta, const float *S0, const void *dout, const void *du,
                                    const float *dS_T, void *dq, void *dk_, void *dv_, void *dalpha, void *dbeta,
                                    float *dS0, int B, int T, int H, int dk, int dv, int variant, int chunk,
                                    int dtype, void *workspace, size_t ws_bytes_given, void *stream,
                                    void *const *events, int n_events) {
    return bwd_timed(q, k, v, alpha, beta, S0, dout, du, dS_T, dq, dk_, dv_, dalpha, dbeta, dS0, B, T, H, dk, dv,
                     variant, chunk, dtype, false, nullptr, 0, workspace, ws_bytes_given, stream, events, n_events);
}

extern "C" int delta_rule_bwd_saved_timed(const void *q, const void *k, const void *v, const void *alpha,
                                          const void *beta, const float *S0, const void *dout, const void *du,
                                          const float *dS_T, void *dq, void *dk_, void *dv_, void *dalpha,
                                          void *dbeta, float *dS0, int B, int T, int H, int dk, int dv, int variant,
                                          int chunk, int dtype, const void *saved, size_t saved_given,
                                          void *workspace, size_t ws_bytes_given, void *stream, void *const *events,
                                          int n_events) {
    return bwd_timed(q, k, v, alpha, beta, S0, dout, du, dS_T, dq, dk_, dv_, dalpha, dbeta, dS0, B, T, H, dk, dv,
                     variant, chunk, dtype, true, saved, saved_given, workspace, ws_bytes_given, stream, events,
                     n_events);
}

extern "C" int delta_rule_launches(int B, int T, int H, int dk, int dv, int variant, int chunk, int dtype,
                                   int for_bwd, const char **names, int max_names) {
    Geo g;
    const int rc = check_shape(B, T, H, dk, dv, variant, chunk, dtype, &g);
    if (rc != DR_OK) return rc;
    if (for_bwd < 0 || for_bwd > 3) return DR_ERR_ARG;
    return launch_plan(g, dtype, for_bwd, names, max_names);
}

extern "C" int delta_rule_plain_launches(int B, int T, int H, int dk, int dv, int variant, int chunk, int dtype,
                                         int for_bwd) {
    Geo g;
    const int rc = check_shape(B, T, H, dk, dv, variant, chunk, dtype, &g);
    if (rc != DR_OK) return rc;
    if (for_bwd < 0 || for_bwd > 3) return DR_ERR_ARG;
    const int n = launch_plan(g, dtype, for_bwd, nullptr, 0);
    if (n <= 0 || T == 0 || (size_t)B * H == 0) return n;
    const bool split = use_split(g, dtype) || use_split_kda(g, dtype, for_bwd) || use_kda_hybrid_bwd(g, dtype, for_bwd);
    const int S = split ? seg_count(g) : 1;
    if (S == 1) return n;
    // in segments: every forward kernel once per segment; the backward's reverse chain and
    // gradient kernel once per segment, the rest once
    return is_bwd(for_bwd) ? n - 2 + 2 * S : n * S;
}

extern "C" int delta_rule_decode(const void *q, const void *k, const void *v, const void *alpha, const void *beta,
                                 const float *S_in, float *S_out, void *out, void *u, int B, int T, int H, int dk,
                                 int dv, int variant, int dtype, void *stream) {
    Geo g;
    int rc = check_shape(B, T, H, dk, dv, variant, 64, dtype, &g);
    if (rc != DR_OK) return rc;
    cudaStream_t s = (cudaStream_t)stream;
    const bool empty = (size_t)B * H == 0;
    if (empty) return DR_OK;
    if (T == 0) return S_out == S_in ? DR_OK : copy_state(S_out, S_in, g, s);
    if (!q || !k || !v || !beta || !out) return DR_ERR_ARG;
    if (variant != DR_DELTANET && !alpha) return DR_ERR_ARG;
    const void *ptrs[] = {q, k, v, variant == DR_KDA ? alpha : nullptr, S_in, S_out, out, u};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return DR_ERR_ALIGN;
    if (!aligned_elem(beta, dtype) || (variant == DR_GATED && !aligned_elem(alpha, dtype))) return DR_ERR_ALIGN;
    Tensors t = {};
    t.q = q; t.k = k; t.v = v; t.alpha = alpha; t.beta = beta; t.S0 = S_in; t.out = out; t.u = u; t.S_T = S_out;
    Rec rec;
    return launch_status(decode_fwd(g, t, dtype == DR_BF16, s, rec));
}

// Shape check shared by the pre/post entry points: rows of d channels.
static int check_rows(int B, int T, int H, int d, int dtype, size_t *rows) {
    if (B < 0 || T < 0 || H < 0 || d <= 0) return DR_ERR_ARG;
    if (dtype != DR_F32 && dtype != DR_BF16) return DR_ERR_ARG;
    if (d != 64 && d != 128) return DR_ERR_UNSUPPORTED;
    if ((double)B * T * H * d > 9.0e18 / 16) return DR_ERR_ARG;
    *rows = (size_t)B * T * H;
    return DR_OK;
}

static int preop_impl(const void *q_raw, const void *k_raw, const void *beta_raw, const void *gate_raw,
                      const void *dq, const void *dk_, const void *dbeta, const void *dloga, void *q, void *k,
                      void *beta, void *loga, int B, int T, int H, int dk, int variant, int dtype, void *stream,
                      bool bwd) {
    size_t rows = 0;
    int rc = check_rows(B, T, H, dk, dtype, &rows);
    if (rc != DR_OK) return rc;
    if (variant < DR_DELTANET || variant > DR_KDA) return DR_ERR_ARG;
    if (rows == 0) return DR_OK;
    const bool gated = variant != DR_DELTANET;
    if (!q_raw || !k_raw || !beta_raw || !q || !k || !beta) return DR_ERR_ARG;
    if (gated && (!gate_raw || !loga)) return DR_ERR_ARG;
    if (bwd && (!dq || !dk_ || !dbeta || (gated && !dloga))) return DR_ERR_ARG;
    const bool kda = variant == DR_KDA;
    const void *vec[] = {q_raw, k_raw, q, k, dq, dk_, kda ? gate_raw : nullptr, kda ? loga : nullptr,
                         kda ? dloga : nullptr};
    for (const void *p : vec)
        if (p && !aligned16(p)) return DR_ERR_ALIGN;
    const void *sca[] = {beta_raw, beta, dbeta, variant == DR_GATED ? gate_raw : nullptr,
                         variant == DR_GATED ? loga : nullptr, variant == DR_GATED ? dloga : nullptr};
    for (const void *p : sca)
        if (p && !aligned_elem(p, dtype)) return DR_ERR_ALIGN;
    PrePost pp = {};
    pp.q = q_raw; pp.k = k_raw; pp.b = beta_raw; pp.a = gated ? gate_raw : nullptr;
    pp.dq = dq; pp.dk = dk_; pp.db = dbeta; pp.da = gated ? dloga : nullptr;
    pp.qo = q; pp.ko = k; pp.bo = beta; pp.ao = gated ? loga : nullptr;
    pp.rows = rows; pp.d = dk; pp.variant = variant;
    return launch_status(preop_run(pp, dtype == DR_BF16, bwd, (cudaStream_t)stream));
}

extern "C" int delta_rule_preop(const void *q_raw, const void *k_raw, const void *beta_raw, const void *gate_raw,
                                void *q, void *k, void *beta, void *loga, int B, int T, int H, int dk, int variant,
                                int dtype, void *stream) {
    return preop_impl(q_raw, k_raw, beta_raw, gate_raw, nullptr, nullptr, nullptr, nullptr, q, k, beta, loga, B, T,
                      H, dk, variant, dtype, stream, false);
}

extern "C" int delta_rule_preop_bwd(const void *q_raw, const void *k_raw, const void *beta_raw,
                                    const void *gate_raw, const void *dq, const void *dk_, const void *dbeta,
                                    const void *dloga, void *dq_raw, void *dk_raw, void *dbeta_raw, void *dgate_raw,
                                    int B, int T, int H, int dk, int variant, int dtype, void *stream) {
    return preop_impl(q_raw, k_raw, beta_raw, gate_raw, dq, dk_, dbeta, dloga, dq_raw, dk_raw, dbeta_raw, dgate_raw,
                      B, T, H, dk, variant, dtype, stream, true);
}

extern "C" size_t delta_rule_postop_workspace_size(int dv) {
    if (dv != 64 && dv != 128) return (size_t)-1;
    return postop_ws_bytes(dv);
}

extern "C" int delta_rule_postop(const void *o, const void *gate, const float *weight, void *y, int B, int T, int H,
                                 int dv, int dtype, void *stream) {
    size_t rows = 0;
    int rc = check_rows(B, T, H, dv, dtype, &rows);
    if (rc != DR_OK) return rc;
    if (rows == 0) return DR_OK;
    if (!o || !gate || !y) return DR_ERR_ARG;
    const void *vec[] = {o, gate, weight, y};
    for (const void *p : vec)
        if (p && !aligned16(p)) return DR_ERR_ALIGN;
    PrePost pp = {};
    pp.q = o; pp.k = gate; pp.w = weight; pp.qo = y; pp.rows = rows; pp.d = dv;
    return launch_status(postop_run(pp, dtype == DR_BF16, false, (cudaStream_t)stream));
}

extern "C" int delta_rule_postop_bwd(const void *o, const void *gate, const float *weight, const void *dy, void *do_,
                                     void *dgate, float *dweight, int B, int T, int H, int dv, int dtype,
                                     void *workspace, size_t ws_bytes_given, void *stream) {
    size_t rows = 0;
    int rc = check_rows(B, T, H, dv, dtype, &rows);
    if (rc != DR_OK) return rc;
    if (!o || !gate || !dy || !do_ || !dgate) return DR_ERR_ARG;
    const void *vec[] = {o, gate, weight, dy, do_, dgate, dweight};
    for (const void *p : vec)
        if (p && !aligned16(p)) return DR_ERR_ALIGN;
    rc = check_buffer(workspace, ws_bytes_given, postop_ws_bytes(dv));
    if (rc != DR_OK) return rc;
    PrePost pp = {};
    pp.q = o; pp.k = gate; pp.w = weight; pp.dq = dy; pp.qo = do_; pp.ko = dgate; pp.dw = dweight;
    pp.part = (float *)workspace; pp.rows = rows; pp.d = dv;
    return launch_status(postop_run(pp, dtype == DR_BF16, true, (cudaStream_t)stream));
}

// Shape check of the short convolution: B sequences of T tokens with D channels.
static int check_conv(int B, int T, int D, int dtype) {
    if (B < 0 || T < 0 || D <= 0) return DR_ERR_ARG;
    if (dtype != DR_F32 && dtype != DR_BF16) return DR_ERR_ARG;
    if (D % 8 != 0) return DR_ERR_UNSUPPORTED;
    if ((double)B * ((double)T + 3) * D > 9.0e18 / 16) return DR_ERR_ARG;
    const bool bf16 = dtype == DR_BF16;
    if (shortconv_ctas(B, T, D, bf16, false) > INT_MAX || shortconv_ctas(B, T, D, bf16, true) > INT_MAX)
        return DR_ERR_UNSUPPORTED;
    return DR_OK;
}

extern "C" size_t delta_rule_shortconv_workspace_size(int B, int T, int D) {
    if (B < 0 || T < 0 || D <= 0 || D % 8 != 0) return (size_t)-1;
    return shortconv_ws_bytes(B, T, D);
}

extern "C" int delta_rule_shortconv(const void *x, const float *w, const void *x_prev, void *y, void *cache_out,
                                    int B, int T, int D, int dtype, void *stream) {
    int rc = check_conv(B, T, D, dtype);
    if (rc != DR_OK) return rc;
    if (B == 0) return DR_OK;
    if (!w || (T > 0 && (!x || !y))) return DR_ERR_ARG;
    const void *vec[] = {x, x_prev, y, cache_out};
    for (const void *p : vec)
        if (p && !aligned16(p)) return DR_ERR_ALIGN;
    if (!aligned_elem(w, DR_F32)) return DR_ERR_ALIGN;
    if (T == 0 && !cache_out) return DR_OK;
    ShortConv sc = {};
    sc.x = x; sc.w = w; sc.cin = x_prev; sc.y = y; sc.cout = cache_out; sc.B = B; sc.T = T; sc.D = D;
    return launch_status(shortconv_run(sc, dtype == DR_BF16, false, (cudaStream_t)stream));
}

extern "C" int delta_rule_shortconv_bwd(const void *x, const float *w, const void *x_prev, const void *dy,
                                        void *dx, float *dw, void *dx_prev, int B, int T, int D, int dtype,
                                        void *workspace, size_t ws_bytes_given, void *stream) {
    int rc = check_conv(B, T, D, dtype);
    if (rc != DR_OK) return rc;
    if (B == 0) return DR_OK;
    if (!w || (T > 0 && (!x || !dy || !dx))) return DR_ERR_ARG;
    const void *vec[] = {x, x_prev, dy, dx, dx_prev};
    for (const void *p : vec)
        if (p && !aligned16(p)) return DR_ERR_ALIGN;
    if (!aligned_elem(w, DR_F32) || (dw && !aligned_elem(dw, DR_F32))) return DR_ERR_ALIGN;
    if (dw) {
        rc = check_buffer(workspace, ws_bytes_given, shortconv_ws_bytes(B, T, D));
        if (rc != DR_OK) return rc;
    }
    if (T == 0 && !dw && !dx_prev) return DR_OK;
    ShortConv sc = {};
    sc.x = x; sc.w = w; sc.cin = x_prev; sc.dy = dy; sc.dx = dx; sc.dw = dw; sc.dcin = dx_prev;
    sc.part = (float *)workspace; sc.B = B; sc.T = T; sc.D = D;
    return launch_status(shortconv_run(sc, dtype == DR_BF16, true, (cudaStream_t)stream));
}

// Shape check of the routing products: M tokens, K = H dv write-value channels, N hidden channels.
static int check_clvr(int M, int K, int N, int dtype) {
    if (M < 0 || K <= 0 || N <= 0) return DR_ERR_ARG;
    if (dtype != DR_F32 && dtype != DR_BF16) return DR_ERR_ARG;
    if (K % 8 != 0 || N % 8 != 0) return DR_ERR_UNSUPPORTED;
    return DR_OK;
}

extern "C" size_t delta_rule_clvr_workspace_size(void) { return clvr_ws_bytes(); }

extern "C" int delta_rule_clvr(const void *u, const void *W, const void *h, void *h_out, int M, int K, int N,
                               int dtype, void *workspace, size_t ws_bytes_given, void *stream) {
    int rc = check_clvr(M, K, N, dtype);
    if (rc != DR_OK || M == 0) return rc;
    if (!u || !W || !h_out) return DR_ERR_ARG;
    const void *vec[] = {u, W, h, h_out};
    for (const void *p : vec)
        if (p && !aligned16(p)) return DR_ERR_ALIGN;
    rc = check_buffer(workspace, ws_bytes_given, clvr_ws_bytes());
    if (rc != DR_OK) return rc;
    return clvr_fwd_run(u, W, h, h_out, M, K, N, dtype == DR_BF16, workspace, ws_bytes_given, (cudaStream_t)stream);
}

extern "C" int delta_rule_clvr_bwd(const void *u, const void *W, const void *dh_out, void *du, float *dW, int M,
                                   int K, int N, int dtype, void *workspace, size_t ws_bytes_given, void *stream) {
    int rc = check_clvr(M, K, N, dtype);
    if (rc != DR_OK) return rc;
    if (!u || !W || !dh_out) return M == 0 ? DR_OK : DR_ERR_ARG;
    const void *vec[] = {u, W, dh_out, du, dW};
    for (const void *p : vec)
        if (p && !aligned16(p)) return DR_ERR_ALIGN;
    if (M == 0) {  // no tokens: dW is an empty sum
        return dW ? launch_status(cudaMemsetAsync(dW, 0, (size_t)K * N * sizeof(float), (cudaStream_t)stream)) : DR_OK;
    }
    rc = check_buffer(workspace, ws_bytes_given, clvr_ws_bytes());
    if (rc != DR_OK) return rc;
    return clvr_bwd_run(u, W, dh_out, du, dW, M, K, N, dtype == DR_BF16, workspace, ws_bytes_given,
                        (cudaStream_t)stream);
}

// Self-test of the bounded waits: one thread waits for an mbarrier phase that nothing
// completes; the wait gives up after limit_ns, raises the device error word and returns.
__global__ void k_selftest_wait(unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);
        abort_flag = 0;
        tc::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) tc::mbar_wait(&bar, 0, &abort_flag, limit_ns);
}

extern "C" int delta_rule_selftest_timeout(unsigned limit_us, void *stream) {
    if (limit_us == 0 || limit_us > 1000000u) return DR_ERR_ARG;
    k_selftest_wait<<<1, 32, 0, (cudaStream_t)stream>>>(1000ull * limit_us);
    return launch_status(cudaGetLastError());
}

extern "C" const char *delta_rule_strerror(int code) {
    switch (code) {
        case DR_OK: return "ok";
        case DR_ERR_ARG: return "invalid argument";
        case DR_ERR_UNSUPPORTED: return "unsupported shape or option";
        case DR_ERR_ALIGN: return "misaligned pointer (16 B; workspace 256 B)";
        case DR_ERR_WORKSPACE: return "workspace missing or too small";
        case DR_ERR_CUDA: return "CUDA error";
        case DR_ERR_TIMEOUT: return "device wait timed out";
        default: return "unknown error code";
    }
}

extern "C" int delta_rule_sync_status(void *stream) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return DR_ERR_CUDA;
    int word = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&word, g_dev_error, sizeof(int)) != cudaSuccess) return DR_ERR_CUDA;
    if (word && cudaMemcpyToSymbol(g_dev_error, &zero, sizeof(int)) != cudaSuccess) return DR_ERR_CUDA;
    return (word & DEVERR_TIMEOUT) ? DR_ERR_TIMEOUT : DR_OK;
}
