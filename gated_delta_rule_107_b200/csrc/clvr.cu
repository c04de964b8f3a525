// clvr.cu -- cross-layer value routing: h_out = h + U W and its gradients.
//
// ETH news page on the architecture study, section 七 (and the explainer's CLVR section): a
// layer's write values u_t = beta_t (v_t - S'_t^T k_t) enter a higher layer's hidden stream, the
// residual stream all layers share, through a projection W that starts at zero.  With U the write
// values as [B*T, H*dv] (the core's u output, unchanged), W [H*dv, D] and h [B*T, D]:
//     h_out = h + U W,      dU = dH W^T,      dW = U^T dH,      dh = dH.
// These are plain dense products, so they run as cuBLASLt GEMMs: bf16 operands on the tensor
// cores with fp32 accumulation (fp32 operands and arithmetic for fp32 I/O), the residual add as
// the GEMM's beta = 1 term, so that h_out is written in the same pass.  The routing step and
// its weight are the model's; the library only needs U, which the core writes anyway.
#include <cublasLt.h>

#include <mutex>

#include "../../include/delta_rule.h"
#include "clvr.cuh"

namespace dr {
namespace clv {

constexpr size_t WS = (size_t)32 << 20;  // cuBLASLt workspace, provided by the caller

// One cuBLASLt handle per process, created on first use (the library's only host-side state).
cublasLtHandle_t handle(bool *ok) {
    static cublasLtHandle_t h = nullptr;
    static cublasStatus_t st = CUBLAS_STATUS_SUCCESS;
    static std::once_flag once;
    std::call_once(once, [] { st = cublasLtCreate(&h); });
    *ok = st == CUBLAS_STATUS_SUCCESS;
    return h;
}

// Row-major D [m][n] = op(A) op(B) + beta C, op(A) [m][k] being A [m][k] or, with ta, the
// transpose of A [k][m]; op(B) [k][n] being B [k][n] or, with tb, the transpose of B [n][k].
// cuBLASLt works column-major, so it forms D^T = op(B)^T op(A)^T from the same buffers.  The
// descriptors and the chosen algorithm of each distinct problem are kept for the process (a
// short list under a mutex), so that a repeated call costs one cublasLtMatmul.
struct Plan {
    int m, n, k, ta, tb, ab, cd;
    size_t wsb;
    cublasLtMatmulDesc_t op;
    cublasLtMatrixLayout_t La, Lb, Lc;
    cublasLtMatmulAlgo_t algo;
};
constexpr int MAX_PLANS = 64;

cublasStatus_t make_plan(cublasLtHandle_t lt, Plan &p) {
    const cublasOperation_t o1 = p.tb ? CUBLAS_OP_T : CUBLAS_OP_N, o2 = p.ta ? CUBLAS_OP_T : CUBLAS_OP_N;
    const cudaDataType_t ab = (cudaDataType_t)p.ab, cd = (cudaDataType_t)p.cd;
    const int m = p.m, n = p.n, k = p.k;
    cublasLtMatmulPreference_t pref = nullptr;
    cublasStatus_t st = cublasLtMatmulDescCreate(&p.op, CUBLAS_COMPUTE_32F, CUDA_R_32F);
    if (st == CUBLAS_STATUS_SUCCESS) st = cublasLtMatmulDescSetAttribute(p.op, CUBLASLT_MATMUL_DESC_TRANSA, &o1, sizeof(o1));
    if (st == CUBLAS_STATUS_SUCCESS) st = cublasLtMatmulDescSetAttribute(p.op, CUBLASLT_MATMUL_DESC_TRANSB, &o2, sizeof(o2));
    // first operand, B: column-major n x k (ld n), or k x n (ld k) read transposed
    if (st == CUBLAS_STATUS_SUCCESS) st = cublasLtMatrixLayoutCreate(&p.La, ab, p.tb ? k : n, p.tb ? n : k, p.tb ? k : n);
    // second operand, A: column-major k x m (ld k), or m x k (ld m) read transposed
    if (st == CUBLAS_STATUS_SUCCESS) st = cublasLtMatrixLayoutCreate(&p.Lb, ab, p.ta ? m : k, p.ta ? k : m, p.ta ? m : k);
    if (st == CUBLAS_STATUS_SUCCESS) st = cublasLtMatrixLayoutCreate(&p.Lc, cd, n, m, n);
    if (st == CUBLAS_STATUS_SUCCESS) st = cublasLtMatmulPreferenceCreate(&pref);
    if (st == CUBLAS_STATUS_SUCCESS)
        st = cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &p.wsb, sizeof(p.wsb));
    cublasLtMatmulHeuristicResult_t res = {};
    int found = 0;
    if (st == CUBLAS_STATUS_SUCCESS)
        st = cublasLtMatmulAlgoGetHeuristic(lt, p.op, p.La, p.Lb, p.Lc, p.Lc, pref, 1, &res, &found);
    if (st == CUBLAS_STATUS_SUCCESS && found == 0) st = CUBLAS_STATUS_NOT_SUPPORTED;
    if (st == CUBLAS_STATUS_SUCCESS) p.algo = res.algo;
    if (pref) cublasLtMatmulPreferenceDestroy(pref);
    return st;
}

void free_plan(Plan &p) {
    if (p.Lc) cublasLtMatrixLayoutDestroy(p.Lc);
    if (p.Lb) cublasLtMatrixLayoutDestroy(p.Lb);
    if (p.La) cublasLtMatrixLayoutDestroy(p.La);
    if (p.op) cublasLtMatmulDescDestroy(p.op);
}

cublasStatus_t gemm(cublasLtHandle_t lt, const void *A, bool ta, const void *B, bool tb, const void *C, void *D,
                    int m, int n, int k, cudaDataType_t ab, cudaDataType_t cd, float beta, void *ws, size_t wsb,
                    cudaStream_t s) {
    static std::mutex mu;
    static Plan plans[MAX_PLANS];
    static int nplans = 0;
    Plan key = {m, n, k, (int)ta, (int)tb, (int)ab, (int)cd, wsb, nullptr, nullptr, nullptr, nullptr, {}};
    const Plan *use = nullptr;
    Plan local = key;
    {
        std::lock_guard<std::mutex> g(mu);
        for (int i = 0; i < nplans && !use; ++i) {
            const Plan &q = plans[i];
            if (q.m == m && q.n == n && q.k == k && q.ta == key.ta && q.tb == key.tb && q.ab == key.ab &&
                q.cd == key.cd && q.wsb == wsb)
                use = &q;
        }
        if (!use && nplans < MAX_PLANS) {
            Plan &q = plans[nplans];
            q = key;
            const cublasStatus_t st = make_plan(lt, q);
            if (st != CUBLAS_STATUS_SUCCESS) {
                free_plan(q);
                return st;
            }
            use = &plans[nplans++];
        }
    }
    if (!use) {  // the list is full: a plan for this call only
        const cublasStatus_t st = make_plan(lt, local);
        if (st != CUBLAS_STATUS_SUCCESS) {
            free_plan(local);
            return st;
        }
    }
    const Plan &p = use ? *use : local;
    const float alpha = 1.f;
    const cublasStatus_t st =
        cublasLtMatmul(lt, p.op, &alpha, B, p.La, A, p.Lb, &beta, C ? C : D, p.Lc, D, p.Lc, &p.algo, ws, wsb, s);
    if (!use) free_plan(local);
    return st;
}

int status(cublasStatus_t st) {
    if (st == CUBLAS_STATUS_SUCCESS) return DR_OK;
    return st == CUBLAS_STATUS_NOT_SUPPORTED ? DR_ERR_UNSUPPORTED : DR_ERR_CUDA;
}

}  // namespace clv

size_t clvr_ws_bytes() { return clv::WS; }

int clvr_fwd_run(const void *U, const void *W, const void *h, void *h_out, int M, int K, int N, bool bf16,
                 void *ws, size_t ws_bytes, cudaStream_t s) {
    bool ok = false;
    cublasLtHandle_t lt = clv::handle(&ok);
    if (!ok) return DR_ERR_CUDA;
    const cudaDataType_t t = bf16 ? CUDA_R_16BF : CUDA_R_32F;
    return clv::status(clv::gemm(lt, U, false, W, false, h, h_out, M, N, K, t, t, h ? 1.f : 0.f, ws, ws_bytes, s));
}

int clvr_bwd_run(const void *U, const void *W, const void *dH, void *dU, float *dW, int M, int K, int N, bool bf16,
                 void *ws, size_t ws_bytes, cudaStream_t s) {
    bool ok = false;
    cublasLtHandle_t lt = clv::handle(&ok);
    if (!ok) return DR_ERR_CUDA;
    const cudaDataType_t t = bf16 ? CUDA_R_16BF : CUDA_R_32F;
    if (dU) {  // dU [M][K] = dH [M][N] W^T, W [K][N]
        const int rc = clv::status(clv::gemm(lt, dH, false, W, true, nullptr, dU, M, K, N, t, t, 0.f, ws, ws_bytes, s));
        if (rc != DR_OK) return rc;
    }
    if (dW)  // dW [K][N] = U^T dH, U [M][K]
        return clv::status(clv::gemm(lt, U, true, dH, false, nullptr, dW, K, N, M, t, CUDA_R_32F, 0.f, ws, ws_bytes, s));
    return DR_OK;
}

}  // namespace dr
