// decode.cu -- the recurrent form of the gated delta rule for short sequences (decoding):
// the state is read once, stepped through the tokens in registers and written once.
//
// Per token, with S' = Diag(alpha_t) S (section 2.1 of "线性注意力架构演进与Kimi Delta
// Attention创新实践"; the write value of the cross-layer routing in the explainer):
//   u_t = beta_t (v_t - S'^T k_t)
//   S   = S' + k_t u_t^T
//   o_t = S^T q_t = S'^T q_t + u_t (k_t . q_t)
// so both column reductions of a step (S'^T k and S'^T q) come from the one decayed state.
//
// One CTA per (b, h, 32 value columns); 128 threads.  Lane l of warp w owns value column
// 8 w + (l & 7) and the key rows (l >> 3) * dk / 4 ... + dk / 4 - 1 of it, so a column's
// sums close with two shuffles and neighbouring lanes touch neighbouring columns.  The
// tokens' q, k (and the KDA gate) are staged in shared memory 16 at a time.
#include "decode.cuh"

namespace dr {
namespace dec {

constexpr int NCOL = 32;  // value columns per CTA
constexpr int TT = 16;    // tokens staged per round

template <typename E, int VAR, int DK>
__global__ void __launch_bounds__(128) k_decode(const E *__restrict__ q, const E *__restrict__ k,
                                                const E *__restrict__ v, const E *__restrict__ alpha,
                                                const E *__restrict__ beta, const float *S_in, float *S_out,
                                                E *__restrict__ out, E *__restrict__ u, int T, int H, int dv) {
    constexpr int RPT = DK / 4;  // key rows per thread
    __shared__ float sq[TT][DK], sk[TT][DK], sa[VAR == VAR_KDA ? TT : 1][DK];
    __shared__ float sv[TT][NCOL], sg[TT], sb[TT];
    const int b = blockIdx.z, h = blockIdx.y, j0 = blockIdx.x * NCOL;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int jl = warp * 8 + (lane & 7), j = j0 + jl, r0 = (lane >> 3) * RPT;
    const size_t head = ((size_t)b * H + h) * DK * dv;

    float s[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) s[i] = S_in ? S_in[head + (size_t)(r0 + i) * dv + j] : 0.f;

    for (int t0 = 0; t0 < T; t0 += TT) {
        const int nt = min(TT, T - t0);
        __syncthreads();  // the previous round's tokens are no longer read
        for (int x = tid; x < nt * DK; x += 128) {
            const int tt = x / DK, c = x - tt * DK;
            const size_t row = ((size_t)b * T + t0 + tt) * H + h;
            sq[tt][c] = to_f(q[row * DK + c]);
            sk[tt][c] = to_f(k[row * DK + c]);
            if (VAR == VAR_KDA) sa[tt][c] = __expf(to_f(alpha[row * DK + c]));
        }
        for (int x = tid; x < nt * NCOL; x += 128) {
            const int tt = x / NCOL, c = x - tt * NCOL;
            sv[tt][c] = to_f(v[(((size_t)b * T + t0 + tt) * H + h) * dv + j0 + c]);
        }
        if (tid < nt) {
            const size_t row = ((size_t)b * T + t0 + tid) * H + h;
            sb[tid] = to_f(beta[row]);
            sg[tid] = VAR == VAR_GATED ? __expf(to_f(alpha[row])) : 1.f;
        }
        __syncthreads();
        for (int tt = 0; tt < nt; ++tt) {
            // S' = Diag(alpha) S, and this thread's parts of S'^T k, S'^T q and k . q
            float pk = 0.f, pq = 0.f, kq = 0.f;
#pragma unroll
            for (int i = 0; i < RPT; ++i) {
                const int c = r0 + i;
                if (VAR == VAR_GATED) s[i] *= sg[tt];
                if (VAR == VAR_KDA) s[i] *= sa[tt][c];
                pk += s[i] * sk[tt][c];
                pq += s[i] * sq[tt][c];
                kq += sk[tt][c] * sq[tt][c];
            }
#pragma unroll
            for (int o = 8; o < 32; o <<= 1) {
                pk += __shfl_xor_sync(0xffffffffu, pk, o);
                pq += __shfl_xor_sync(0xffffffffu, pq, o);
                kq += __shfl_xor_sync(0xffffffffu, kq, o);
            }
            const float uj = sb[tt] * (sv[tt][jl] - pk);
            const float oj = pq + uj * kq;
#pragma unroll
            for (int i = 0; i < RPT; ++i) s[i] += sk[tt][r0 + i] * uj;
            if (lane < 8) {
                const size_t o_at = (((size_t)b * T + t0 + tt) * H + h) * dv + j;
                out[o_at] = from_f<E>(oj);
                if (u) u[o_at] = from_f<E>(uj);
            }
        }
    }
    if (S_out) {
#pragma unroll
        for (int i = 0; i < RPT; ++i) S_out[head + (size_t)(r0 + i) * dv + j] = s[i];
    }
}

template <typename E, int VAR>
static cudaError_t launch_v(const Geo &g, const Tensors &t, cudaStream_t st) {
    const dim3 grid(g.dv / NCOL, g.H, g.B);
    const E *q = (const E *)t.q, *k = (const E *)t.k, *v = (const E *)t.v, *a = (const E *)t.alpha,
            *bt = (const E *)t.beta;
    if (g.dk == 128)
        k_decode<E, VAR, 128><<<grid, 128, 0, st>>>(q, k, v, a, bt, t.S0, t.S_T, (E *)t.out, (E *)t.u, g.T, g.H, g.dv);
    else
        k_decode<E, VAR, 64><<<grid, 128, 0, st>>>(q, k, v, a, bt, t.S0, t.S_T, (E *)t.out, (E *)t.u, g.T, g.H, g.dv);
    return cudaGetLastError();
}

template <typename E>
static cudaError_t launch_e(const Geo &g, const Tensors &t, cudaStream_t st) {
    if (g.variant == VAR_GATED) return launch_v<E, VAR_GATED>(g, t, st);
    if (g.variant == VAR_KDA) return launch_v<E, VAR_KDA>(g, t, st);
    return launch_v<E, VAR_DELTANET>(g, t, st);
}

}  // namespace dec

// Token-by-token forward (t.S0 -> t.S_T, which may be the same buffer).
cudaError_t decode_fwd(const Geo &g, const Tensors &t, bool bf16, cudaStream_t s, Rec &rec) {
    rec.mark(s);
    return bf16 ? dec::launch_e<__nv_bfloat16>(g, t, s) : dec::launch_e<float>(g, t, s);
}

}  // namespace dr
