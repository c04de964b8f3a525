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
// One CTA per (b, h, 32 value columns); 128 threads.  Thread t owns the 4 value columns
// 4 (t % 8) ... + 3 of the CTA's 32 and the key rows (t / 8) dk / 16 ... + dk / 16 - 1, so
// the state moves as 16-byte rows; a column's sums close with two shuffles inside the warp
// and one exchange through shared memory across the four warps (double-buffered by token,
// so one barrier per token).  The tokens' q, k (and the KDA gate) are staged in shared
// memory 16 at a time.
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
    constexpr int RPT = DK / 16;  // key rows per thread
    __shared__ float sq[TT][DK], sk[TT][DK], sa[VAR == VAR_KDA ? TT : 1][DK];
    __shared__ float sv[TT][NCOL], sg[TT], sb[TT];
    __shared__ float red[2][4][8][9];  // per token parity, warp, column group: S'^T k (4), S'^T q (4), k . q
    const int b = blockIdx.z, h = blockIdx.y, j0 = blockIdx.x * NCOL;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rg = tid >> 3, cg = tid & 7, r0 = rg * RPT, jc = j0 + 4 * cg;
    const size_t head = ((size_t)b * H + h) * DK * dv;

    float s[RPT][4];
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (S_in) x = *reinterpret_cast<const float4 *>(S_in + head + (size_t)(r0 + i) * dv + jc);
        s[i][0] = x.x; s[i][1] = x.y; s[i][2] = x.z; s[i][3] = x.w;
    }

    int par = 0;
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
        for (int tt = 0; tt < nt; ++tt, par ^= 1) {
            // S' = Diag(alpha) S, and this thread's parts of S'^T k, S'^T q (4 columns) and k . q
            float pk[4] = {0.f, 0.f, 0.f, 0.f}, pq[4] = {0.f, 0.f, 0.f, 0.f}, kq = 0.f;
#pragma unroll
            for (int i = 0; i < RPT; ++i) {
                const int c = r0 + i;
                const float kc = sk[tt][c], qc = sq[tt][c];
                const float f = VAR == VAR_GATED ? sg[tt] : (VAR == VAR_KDA ? sa[tt][c] : 1.f);
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    if (VAR != VAR_DELTANET) s[i][jj] *= f;
                    pk[jj] += s[i][jj] * kc;
                    pq[jj] += s[i][jj] * qc;
                }
                kq += kc * qc;
            }
            // sum over the four row groups of this warp (lanes 8 and 16 apart), then over warps
#pragma unroll
            for (int o = 8; o < 32; o <<= 1) {
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    pk[jj] += __shfl_xor_sync(0xffffffffu, pk[jj], o);
                    pq[jj] += __shfl_xor_sync(0xffffffffu, pq[jj], o);
                }
                kq += __shfl_xor_sync(0xffffffffu, kq, o);
            }
            if (lane < 8) {
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    red[par][warp][cg][jj] = pk[jj];
                    red[par][warp][cg][4 + jj] = pq[jj];
                }
                red[par][warp][cg][8] = kq;
            }
            __syncthreads();
            float tk[4] = {0.f, 0.f, 0.f, 0.f}, tq[4] = {0.f, 0.f, 0.f, 0.f}, tkq = 0.f;
#pragma unroll
            for (int wp = 0; wp < 4; ++wp) {
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    tk[jj] += red[par][wp][cg][jj];
                    tq[jj] += red[par][wp][cg][4 + jj];
                }
                tkq += red[par][wp][cg][8];
            }
            float uj[4], oj[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                uj[jj] = sb[tt] * (sv[tt][4 * cg + jj] - tk[jj]);
                oj[jj] = tq[jj] + uj[jj] * tkq;
            }
#pragma unroll
            for (int i = 0; i < RPT; ++i) {
                const float kc = sk[tt][r0 + i];
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) s[i][jj] += kc * uj[jj];
            }
            if (rg == 0) {
                const size_t o_at = (((size_t)b * T + t0 + tt) * H + h) * dv + jc;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    out[o_at + jj] = from_f<E>(oj[jj]);
                    if (u) u[o_at + jj] = from_f<E>(uj[jj]);
                }
            }
        }
    }
    if (S_out) {
#pragma unroll
        for (int i = 0; i < RPT; ++i)
            *reinterpret_cast<float4 *>(S_out + head + (size_t)(r0 + i) * dv + jc) =
                make_float4(s[i][0], s[i][1], s[i][2], s[i][3]);
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
