// simt_path.cu -- chunkwise gated delta rule on CUDA cores, fp32 arithmetic.
//
// This path serves fp32 I/O (where the result must agree with fp64 to ~1e-4,
// beyond what bf16 tensor-core operands allow) and every shape the tensor-core
// path does not specialise.  It follows the chunked form of the recurrence of
// "线性注意力架构演进与Kimi Delta Attention创新实践" section 2.1, solved per chunk
// with the UT transform of section 6.2 and log-space cumulative gates of
// section 7.1.  For one (b, h) and chunk of C tokens with incoming state S:
//
//   g_r   = sum_{i<=r} log alpha_i          (per channel; broadcast for Gated)
//   A_ri  = beta_r sum_c k_rc k_ic e^{g_rc - g_ic}          (i < r)
//   P_ri  =        sum_c q_rc k_ic e^{g_rc - g_ic}          (i <= r)
//   W     = (I+A)^-1 diag(beta) (e^{g} .* K),  U~ = (I+A)^-1 diag(beta) V
//   U     = U~ - W S                  (rows are the write values u_t)
//   O     = (e^{g} .* Q) S + P U
//   S+    = Diag(e^{g_C}) S + (K .* e^{g_C - g})^T U
//
// Every exponent above is of a non-positive number when log alpha <= 0, so no
// intermediate can overflow.  The one split exponential is in the backward at C = 64:
// e^{g_r - g_i} = e^{g_r - m} e^{m - g_i} around a midpoint m of the chunk's gates, used
// only where every channel's gates span at most 120 nats in that chunk (each factor within
// e^{+-60}); other chunks take the direct form.
//
// Kernels (one CTA of 256 threads each):
//   k_prep        grid (N, H, B)     g, A, P, then W and U~ by forward substitution
//   k_scan        grid (dv/32, H, B) serial state chain over chunks, U, S_n
//   k_out         grid (N, H, B)     O = Qtil S_n + P U
//   k_scan_bwd    grid (dv/32, H, B) reverse chain: dU_n and dS_{n+1}
//   k_bwd_state   grid (N, H, B)     dO S^T, -dU S^T, U dS+^T, rowsum(S .* dS+)
//   k_bwd_intra   grid (N, H, B)     everything inside the chunk -> dq dk dv dbeta dlog-alpha
#include "simt_path.cuh"

namespace dr {

static constexpr int NT = 256;  // threads per CTA
static constexpr int JB = 32;   // dv columns per CTA in the scans

template <typename TI> struct IO {
    const TI *q, *k, *v, *alpha, *beta, *dout, *du;
    TI *out, *u, *dq, *dk, *dv, *dalpha, *dbeta;
};

template <typename TI> static IO<TI> io_of(const Tensors &t) {
    IO<TI> x;
    x.q = (const TI *)t.q; x.k = (const TI *)t.k; x.v = (const TI *)t.v;
    x.alpha = (const TI *)t.alpha; x.beta = (const TI *)t.beta;
    x.dout = (const TI *)t.dout; x.du = (const TI *)t.du;
    x.out = (TI *)t.out; x.u = (TI *)t.u; x.dq = (TI *)t.dq; x.dk = (TI *)t.dk; x.dv = (TI *)t.dv;
    x.dalpha = (TI *)t.dalpha; x.dbeta = (TI *)t.dbeta;
    return x;
}

// raw log gate of token row `row`, channel c (0 for DeltaNet)
template <typename TI>
__device__ __forceinline__ float raw_gate(const Geo &g, const TI *alpha, size_t row, int c) {
    if (g.variant == VAR_KDA) return to_f(alpha[row * g.dk + c]);
    if (g.variant == VAR_GATED) return to_f(alpha[row]);
    return 0.f;
}

// ---------------------------------------------------------------------------------------------
// k_prep: per chunk, cumulative gates, A and P, then W and U~ by forward substitution.
// smem: ks, qs, gs [C][dk]; vs [C][dv]; Am, Pm [C][C]; bs [C]
template <typename TI>
__global__ void __launch_bounds__(NT) k_prep(Geo g, IO<TI> io, SimtWs w) {
    const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int C = g.C, DK = g.dk, DV = g.dv;
    const int t0 = n * C, L = min(C, g.T - t0);
    extern __shared__ float sm[];
    float *ks = sm, *qs = ks + C * DK, *gs = qs + C * DK, *vs = gs + C * DK;
    float *Am = vs + C * DV, *Pm = Am + C * C, *bs = Pm + C * C;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    for (int x = tid; x < C * DK; x += NT) {
        const int r = x / DK, c = x % DK;
        float kv = 0.f, qv = 0.f, gv = 0.f;
        if (r < L) {
            const size_t row = g.row(b, t0 + r, h);
            kv = to_f(io.k[row * DK + c]);
            qv = to_f(io.q[row * DK + c]);
            gv = raw_gate(g, io.alpha, row, c);
        }
        ks[x] = kv; qs[x] = qv; gs[x] = gv;
    }
    for (int x = tid; x < C * DV; x += NT) {
        const int r = x / DV, j = x % DV;
        vs[x] = r < L ? to_f(io.v[g.row(b, t0 + r, h) * DV + j]) : 0.f;
    }
    for (int r = tid; r < C; r += NT) bs[r] = r < L ? to_f(io.beta[g.row(b, t0 + r, h)]) : 0.f;
    __syncthreads();
    for (int c = tid; c < DK; c += NT)
        for (int r = 1; r < C; ++r) gs[r * DK + c] += gs[(r - 1) * DK + c];
    __syncthreads();

    // A (strictly lower) and P (lower incl. diagonal), one warp per row
    for (int r = warp; r < C; r += NT / 32) {
        for (int i = 0; i < C; ++i) {
            float a = 0.f, p = 0.f;
            if (i <= r) {
                if (g.variant == VAR_KDA) {
                    for (int c = lane; c < DK; c += 32) {
                        const float e = __expf(gs[r * DK + c] - gs[i * DK + c]);
                        const float kic = ks[i * DK + c] * e;
                        a += ks[r * DK + c] * kic;
                        p += qs[r * DK + c] * kic;
                    }
                } else {
                    for (int c = lane; c < DK; c += 32) {
                        a += ks[r * DK + c] * ks[i * DK + c];
                        p += qs[r * DK + c] * ks[i * DK + c];
                    }
                }
                a = warp_sum(a);
                p = warp_sum(p);
                if (g.variant == VAR_GATED) {
                    const float e = __expf(gs[r * DK] - gs[i * DK]);
                    a *= e;
                    p *= e;
                }
            }
            if (lane == 0) {
                Am[r * C + i] = (i < r) ? bs[r] * a : 0.f;
                Pm[r * C + i] = p;
            }
        }
    }
    __syncthreads();
    {
        const size_t ci = g.chunk(b, h, n);
        float *Pg = w.P + ci * C * C;
        for (int x = tid; x < C * C; x += NT) Pg[x] = Pm[x];
        float *Gg = w.G + ci * C * DK;
        for (int x = tid; x < C * DK; x += NT) Gg[x] = gs[x];
    }
    // right-hand sides: beta e^{g} k and beta v
    for (int x = tid; x < C * DK; x += NT) ks[x] *= bs[x / DK] * __expf(gs[x]);
    for (int x = tid; x < C * DV; x += NT) vs[x] *= bs[x / DV];
    __syncthreads();
    // forward substitution (I + A) X = R, one thread per column of [W | U~]
    for (int x = tid; x < DK + DV; x += NT) {
        float *col = x < DK ? ks + x : vs + (x - DK);
        const int ld = x < DK ? DK : DV;
        for (int r = 1; r < C; ++r) {
            float acc = col[r * ld];
            for (int i = 0; i < r; ++i) acc -= Am[r * C + i] * col[i * ld];
            col[r * ld] = acc;
        }
    }
    __syncthreads();
    {
        const size_t ci = g.chunk(b, h, n);
        float *Wg = w.W + ci * C * DK;
        for (int x = tid; x < C * DK; x += NT) Wg[x] = ks[x];
        float *Ug = w.Ut + ci * C * DV;
        for (int x = tid; x < C * DV; x += NT) Ug[x] = vs[x];
    }
}

// ---------------------------------------------------------------------------------------------
// k_scan: serial over chunks for one (b, h) and 32 state columns.
// smem: S [dk][JB]; Ws, Kb [C][dk]; Us [C][JB]; gam [dk]
template <typename TI>
__global__ void __launch_bounds__(NT) k_scan(Geo g, IO<TI> io, SimtWs w, const float *S0, float *ST, int write_u) {
    const int j0 = blockIdx.x * JB, h = blockIdx.y, b = blockIdx.z;
    const int C = g.C, DK = g.dk, DV = g.dv;
    extern __shared__ float sm[];
    float *S = sm, *Ws = S + DK * JB, *Kb = Ws + C * DK, *Us = Kb + C * DK, *gam = Us + C * JB;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t soff = ((size_t)b * g.H + h) * DK * DV;

    for (int x = tid; x < DK * JB; x += NT) {
        const int c = x / JB, j = x % JB;
        S[x] = S0 ? S0[soff + (size_t)c * DV + j0 + j] : 0.f;
    }
    for (int n = 0; n < g.N; ++n) {
        const int t0 = n * C, L = min(C, g.T - t0);
        const size_t ci = g.chunk(b, h, n);
        const float *Wg = w.W + ci * C * DK, *Gg = w.G + ci * C * DK, *Ug = w.Ut + ci * C * DV;
        __syncthreads();
        for (int x = tid; x < C * DK; x += NT) {
            const int r = x / DK, c = x % DK;
            Ws[x] = Wg[x];
            const float kv = r < L ? to_f(io.k[g.row(b, t0 + r, h) * DK + c]) : 0.f;
            Kb[x] = kv * __expf(Gg[(C - 1) * DK + c] - Gg[x]);
        }
        for (int c = tid; c < DK; c += NT) gam[c] = __expf(Gg[(C - 1) * DK + c]);
        for (int x = tid; x < C * JB; x += NT) Us[x] = Ug[(x / JB) * DV + j0 + (x % JB)];
        {
            float *Sg = w.Sn + ci * DK * DV;
            for (int x = tid; x < DK * JB; x += NT) Sg[(x / JB) * DV + j0 + (x % JB)] = S[x];
        }
        __syncthreads();
        // U = U~ - W S
        for (int r = warp; r < C; r += NT / 32) {
            float acc = Us[r * JB + lane];
            for (int c = 0; c < DK; ++c) acc -= Ws[r * DK + c] * S[c * JB + lane];
            Us[r * JB + lane] = acc;
            w.Un[(ci * C + r) * DV + j0 + lane] = acc;
            if (write_u && r < L) io.u[g.row(b, t0 + r, h) * DV + j0 + lane] = from_f<TI>(acc);
        }
        __syncthreads();
        // S <- Diag(gamma_C) S + Kbar^T U
        for (int c = warp; c < DK; c += NT / 32) {
            float acc = gam[c] * S[c * JB + lane];
            for (int r = 0; r < C; ++r) acc += Kb[r * DK + c] * Us[r * JB + lane];
            S[c * JB + lane] = acc;
        }
    }
    __syncthreads();
    if (ST)
        for (int x = tid; x < DK * JB; x += NT) ST[soff + (size_t)(x / JB) * DV + j0 + (x % JB)] = S[x];
}

// ---------------------------------------------------------------------------------------------
// k_out: O = Qtil S_n + P U for one chunk.
// smem: Qs [C][dk]; Pm [C][C]; Sb [dk][JB]; Ub [C][JB]
template <typename TI>
__global__ void __launch_bounds__(NT) k_out(Geo g, IO<TI> io, SimtWs w) {
    const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int C = g.C, DK = g.dk, DV = g.dv;
    const int t0 = n * C, L = min(C, g.T - t0);
    extern __shared__ float sm[];
    float *Qs = sm, *Pm = Qs + C * DK, *Sb = Pm + C * C, *Ub = Sb + DK * JB;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t ci = g.chunk(b, h, n);
    const float *Gg = w.G + ci * C * DK;
    for (int x = tid; x < C * DK; x += NT) {
        const int r = x / DK, c = x % DK;
        Qs[x] = r < L ? to_f(io.q[g.row(b, t0 + r, h) * DK + c]) * __expf(Gg[x]) : 0.f;
    }
    for (int x = tid; x < C * C; x += NT) Pm[x] = w.P[ci * C * C + x];
    for (int jb = 0; jb < DV; jb += JB) {
        __syncthreads();
        for (int x = tid; x < DK * JB; x += NT) Sb[x] = w.Sn[ci * DK * DV + (size_t)(x / JB) * DV + jb + (x % JB)];
        for (int x = tid; x < C * JB; x += NT) Ub[x] = w.Un[(ci * C + x / JB) * DV + jb + (x % JB)];
        __syncthreads();
        for (int r = warp; r < L; r += NT / 32) {
            float acc = 0.f;
            for (int c = 0; c < DK; ++c) acc += Qs[r * DK + c] * Sb[c * JB + lane];
            for (int i = 0; i <= r; ++i) acc += Pm[r * C + i] * Ub[i * JB + lane];
            io.out[g.row(b, t0 + r, h) * DV + jb + lane] = from_f<TI>(acc);
        }
    }
}

// ---------------------------------------------------------------------------------------------
// k_scan_bwd: reverse chain over chunks for one (b, h) and 32 columns:
//   dU_n = du_n + P^T dO_n + Kbar dS_{n+1};  dS_n = Diag(gamma_C) dS_{n+1} + Qtil^T dO_n - W^T dU_n
// smem: dS [dk][JB]; Qs, Ws, Kb [C][dk]; Pm [C][C]; dOs, dUs [C][JB]; gam [dk]
template <typename TI>
__global__ void __launch_bounds__(NT) k_scan_bwd(Geo g, IO<TI> io, SimtWs w, const float *dST, float *dS0) {
    const int j0 = blockIdx.x * JB, h = blockIdx.y, b = blockIdx.z;
    const int C = g.C, DK = g.dk, DV = g.dv;
    extern __shared__ float sm[];
    float *dS = sm, *Qs = dS + DK * JB, *Ws = Qs + C * DK, *Kb = Ws + C * DK, *Pm = Kb + C * DK;
    float *dOs = Pm + C * C, *dUs = dOs + C * JB, *gam = dUs + C * JB;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t soff = ((size_t)b * g.H + h) * DK * DV;
    for (int x = tid; x < DK * JB; x += NT) dS[x] = dST ? dST[soff + (size_t)(x / JB) * DV + j0 + (x % JB)] : 0.f;
    for (int n = g.N - 1; n >= 0; --n) {
        const int t0 = n * C, L = min(C, g.T - t0);
        const size_t ci = g.chunk(b, h, n);
        const float *Wg = w.W + ci * C * DK, *Gg = w.G + ci * C * DK;
        __syncthreads();
        for (int x = tid; x < C * DK; x += NT) {
            const int r = x / DK, c = x % DK;
            float qv = 0.f, kv = 0.f;
            if (r < L) {
                const size_t row = g.row(b, t0 + r, h);
                qv = to_f(io.q[row * DK + c]);
                kv = to_f(io.k[row * DK + c]);
            }
            Qs[x] = qv * __expf(Gg[x]);
            Kb[x] = kv * __expf(Gg[(C - 1) * DK + c] - Gg[x]);
            Ws[x] = Wg[x];
        }
        for (int c = tid; c < DK; c += NT) gam[c] = __expf(Gg[(C - 1) * DK + c]);
        for (int x = tid; x < C * C; x += NT) Pm[x] = w.P[ci * C * C + x];
        for (int x = tid; x < C * JB; x += NT) {
            const int r = x / JB, j = x % JB;
            float o = 0.f, uu = 0.f;
            if (r < L) {
                const size_t row = g.row(b, t0 + r, h);
                o = io.dout ? to_f(io.dout[row * DV + j0 + j]) : 0.f;
                uu = io.du ? to_f(io.du[row * DV + j0 + j]) : 0.f;
            }
            dOs[x] = o;
            dUs[x] = uu;
        }
        {
            float *dSg = w.dSn + ci * DK * DV;
            for (int x = tid; x < DK * JB; x += NT) dSg[(x / JB) * DV + j0 + (x % JB)] = dS[x];
        }
        __syncthreads();
        for (int r = warp; r < C; r += NT / 32) {
            float acc = dUs[r * JB + lane];
            for (int rr = r; rr < C; ++rr) acc += Pm[rr * C + r] * dOs[rr * JB + lane];
            for (int c = 0; c < DK; ++c) acc += Kb[r * DK + c] * dS[c * JB + lane];
            dUs[r * JB + lane] = acc;
            w.dUn[(ci * C + r) * DV + j0 + lane] = acc;
        }
        __syncthreads();
        for (int c = warp; c < DK; c += NT / 32) {
            float acc = gam[c] * dS[c * JB + lane];
            for (int r = 0; r < C; ++r) acc += Qs[r * DK + c] * dOs[r * JB + lane] - Ws[r * DK + c] * dUs[r * JB + lane];
            dS[c * JB + lane] = acc;
        }
    }
    __syncthreads();
    if (dS0)
        for (int x = tid; x < DK * JB; x += NT) dS0[soff + (size_t)(x / JB) * DV + j0 + (x % JB)] = dS[x];
}

// ---------------------------------------------------------------------------------------------
// k_bwd_state: the chunk's products with S_n and dS_{n+1}:
//   Qd = dO S^T,  dWm = -dU S^T,  Tm = U dS+^T  ([C][dk] each),  RS = rowsum(S .* dS+)  ([dk])
// The direct form, for chunk lengths below 64: one output per thread and step.
// smem: Qd, dWm, Tm [C][dk]; Sb, dSb [dk][JB+1]; dOb, dUb, Ub [C][JB]; rs [dk]
template <typename TI>
__device__ __forceinline__ void state_direct(const Geo &g, const IO<TI> &io, const SimtWs &w) {
    const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int C = g.C, DK = g.dk, DV = g.dv;
    const int t0 = n * C, L = min(C, g.T - t0);
    constexpr int LD = JB + 1;
    extern __shared__ float sm[];
    float *Qd = sm, *dWm = Qd + C * DK, *Tm = dWm + C * DK, *Sb = Tm + C * DK, *dSb = Sb + DK * LD;
    float *dOb = dSb + DK * LD, *dUb = dOb + C * JB, *Ub = dUb + C * JB, *rs = Ub + C * JB;
    const int tid = threadIdx.x;
    const size_t ci = g.chunk(b, h, n);
    for (int x = tid; x < C * DK; x += NT) Qd[x] = dWm[x] = Tm[x] = 0.f;
    for (int c = tid; c < DK; c += NT) rs[c] = 0.f;
    for (int jb = 0; jb < DV; jb += JB) {
        __syncthreads();
        for (int x = tid; x < DK * JB; x += NT) {
            const int c = x / JB, j = x % JB;
            Sb[c * LD + j] = w.Sn[ci * DK * DV + (size_t)c * DV + jb + j];
            dSb[c * LD + j] = w.dSn[ci * DK * DV + (size_t)c * DV + jb + j];
        }
        for (int x = tid; x < C * JB; x += NT) {
            const int r = x / JB, j = x % JB;
            dOb[x] = (r < L && io.dout) ? to_f(io.dout[g.row(b, t0 + r, h) * DV + jb + j]) : 0.f;
            dUb[x] = w.dUn[(ci * C + r) * DV + jb + j];
            Ub[x] = w.Un[(ci * C + r) * DV + jb + j];
        }
        __syncthreads();
        for (int x = tid; x < C * DK; x += NT) {
            const int r = x / DK, c = x % DK;
            float a1 = 0.f, a2 = 0.f, a3 = 0.f;
            for (int j = 0; j < JB; ++j) {
                const float s = Sb[c * LD + j];
                a1 += dOb[r * JB + j] * s;
                a2 += dUb[r * JB + j] * s;
                a3 += Ub[r * JB + j] * dSb[c * LD + j];
            }
            Qd[x] += a1;
            dWm[x] -= a2;
            Tm[x] += a3;
        }
        for (int c = tid; c < DK; c += NT) {
            float a = 0.f;
            for (int j = 0; j < JB; ++j) a += Sb[c * LD + j] * dSb[c * LD + j];
            rs[c] += a;
        }
    }
    __syncthreads();
    for (int x = tid; x < C * DK; x += NT) {
        w.Qd[ci * C * DK + x] = Qd[x];
        w.dWm[ci * C * DK + x] = dWm[x];
        w.Tm[ci * C * DK + x] = Tm[x];
    }
    for (int c = tid; c < DK; c += NT) w.RS[ci * DK + c] = rs[c];
}

// cp.async (4-byte) copies, global to shared, in commit groups
__device__ __forceinline__ void cp_async4(float *dst, const float *src) {
    const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;\n" ::: "memory"); }

// At C = 64: thread t keeps a 4 x (dk / 16) block of all three products in registers (rows
// 4 (t / 16) .. + 3, columns t % 16 + 16 v), and dv passes through shared memory JB columns at a
// time, double-buffered: the next block's fp32 operands are copied asynchronously (and its dO
// rows loaded into registers) while the current block is multiplied.
// smem, two stages of: Sb, dSb [dk][JB+1]; dOb, dUb, Ub [64][JB+1]
template <typename TI, int DK>
__device__ __forceinline__ void state_tiled(const Geo &g, const IO<TI> &io, const SimtWs &w) {
    constexpr int C = 64, CW = DK / 16, LD = JB + 1, STG = (2 * DK + 3 * C) * LD, PO = C * JB / NT;
    static_assert(NT == 256, "16 x 16 thread blocks");
    const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int DV = g.dv, t0 = n * C, L = min(C, g.T - t0), R = DV / JB;
    extern __shared__ float sm[];
    const int tid = threadIdx.x;
    const size_t ci = g.chunk(b, h, n);
    const int r0 = 4 * (tid >> 4), cb = tid & 15;
    auto issue = [&](int it, float *st) {
        const int jb = it * JB;
        float *Sb = st, *dSb = Sb + DK * LD, *dUb = dSb + DK * LD + C * LD, *Ub = dUb + C * LD;
        for (int x = tid; x < DK * JB; x += NT) {
            const int c = x / JB, j = x % JB;
            const size_t src = ci * DK * DV + (size_t)c * DV + jb + j;
            cp_async4(Sb + c * LD + j, w.Sn + src);
            cp_async4(dSb + c * LD + j, w.dSn + src);
        }
        for (int x = tid; x < C * JB; x += NT) {
            const int r = x / JB, j = x % JB;
            const size_t src = (ci * C + r) * DV + jb + j;
            cp_async4(dUb + r * LD + j, w.dUn + src);
            cp_async4(Ub + r * LD + j, w.Un + src);
        }
    };
    float od[PO];
    auto fetch_do = [&](int it) {
#pragma unroll
        for (int e = 0; e < PO; ++e) {
            const int x = tid + e * NT, r = x / JB, j = x % JB;
            od[e] = io.dout ? to_f(io.dout[g.row(b, t0 + min(r, L - 1), h) * DV + it * JB + j]) : 0.f;
        }
    };
    auto store_do = [&](float *st) {
        float *dOb = st + 2 * DK * LD;
#pragma unroll
        for (int e = 0; e < PO; ++e) {
            const int x = tid + e * NT, r = x / JB, j = x % JB;
            dOb[r * LD + j] = r < L ? od[e] : 0.f;
        }
    };
    float qd[4][CW], dw[4][CW], tm[4][CW];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < CW; ++v) qd[u][v] = dw[u][v] = tm[u][v] = 0.f;
    float rs = 0.f;
    issue(0, sm);
    cp_async_commit();
    fetch_do(0);
    store_do(sm);
    for (int it = 0; it < R; ++it) {
        float *cur = sm + (it & 1) * STG, *oth = sm + ((it + 1) & 1) * STG;
        if (it + 1 < R) {
            issue(it + 1, oth);
            fetch_do(it + 1);
        }
        cp_async_commit();
        cp_async_wait1();  // all groups but the newest: block it has landed
        __syncthreads();
        const float *Sb = cur, *dSb = Sb + DK * LD, *dOb = dSb + DK * LD, *dUb = dOb + C * LD, *Ub = dUb + C * LD;
#pragma unroll 2
        for (int j = 0; j < JB; ++j) {
            float ao[4], ad[4], au[4], bS[CW], bD[CW];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                ao[u] = dOb[(r0 + u) * LD + j];
                ad[u] = dUb[(r0 + u) * LD + j];
                au[u] = Ub[(r0 + u) * LD + j];
            }
#pragma unroll
            for (int v = 0; v < CW; ++v) {
                bS[v] = Sb[(cb + 16 * v) * LD + j];
                bD[v] = dSb[(cb + 16 * v) * LD + j];
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < CW; ++v) {
                    qd[u][v] += ao[u] * bS[v];
                    dw[u][v] += ad[u] * bS[v];
                    tm[u][v] += au[u] * bD[v];
                }
        }
        if (tid < DK)
            for (int j = 0; j < JB; ++j) rs += Sb[tid * LD + j] * dSb[tid * LD + j];
        if (it + 1 < R) store_do(oth);
        __syncthreads();  // the current stage is refilled next
    }
    const size_t base = ci * C * DK;
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < CW; ++v) {
            const size_t x = base + (size_t)(r0 + u) * DK + cb + 16 * v;
            w.Qd[x] = qd[u][v];
            w.dWm[x] = -dw[u][v];
            w.Tm[x] = tm[u][v];
        }
    if (tid < DK) w.RS[ci * DK + tid] = rs;
}

template <typename TI>
__global__ void __launch_bounds__(NT) k_bwd_state(Geo g, IO<TI> io, SimtWs w) {
    if (g.C == 64) {
        if (g.dk == 128) state_tiled<TI, 128>(g, io, w);
        else state_tiled<TI, 64>(g, io, w);
    } else {
        state_direct<TI>(g, io, w);
    }
}

// ---------------------------------------------------------------------------------------------
// k_bwd_intra: all remaining gradients of one chunk.
//   [dB_k | dB_v] = (I+A)^-T [dW | dU]                         (back substitution)
//   dA_ri = -(dB_k,r . W_i + dB_v,r . U~_i)  (i<r);  dM = diag(beta) dA
//   dP_ri = dO_r . U_i  (i<=r)
//   then the gradients through e^{g} q, e^{g} k, k e^{-g} pairs, k e^{g_C - g}, e^{g_C},
//   beta, and the reverse in-chunk cumsum of dg into d log alpha.
// This direct form takes one exponential per (row, pair, channel) and serves every chunk length;
// at C = 64 it runs only for KDA chunks whose gates span more than the factorised form below
// accepts.
// smem: ks, qs, gs [C][dk]; Y [C][dk+dv]; M, dM, dP [C][C]; bs, dbs, red [C]
template <typename TI>
__device__ __forceinline__ void intra_direct(const Geo &g, const IO<TI> &io, const SimtWs &w) {
    const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int C = g.C, DK = g.dk, DV = g.dv, DY = g.dk + g.dv;
    const int t0 = n * C, L = min(C, g.T - t0);
    extern __shared__ float sm[];
    float *ks = sm, *qs = ks + C * DK, *gs = qs + C * DK, *Y = gs + C * DK;
    float *M = Y + C * DY, *dM = M + C * C, *dP = dM + C * C, *bs = dP + C * C, *dbs = bs + C, *red = dbs + C;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool kda = g.variant == VAR_KDA;
    const size_t ci = g.chunk(b, h, n);
    const float *Gg = w.G + ci * C * DK;

    for (int x = tid; x < C * DK; x += NT) {
        const int r = x / DK, c = x % DK;
        float kv = 0.f, qv = 0.f;
        if (r < L) {
            const size_t row = g.row(b, t0 + r, h);
            kv = to_f(io.k[row * DK + c]);
            qv = to_f(io.q[row * DK + c]);
        }
        ks[x] = kv; qs[x] = qv; gs[x] = Gg[x];
        Y[r * DY + c] = w.dWm[ci * C * DK + x];
    }
    for (int x = tid; x < C * DV; x += NT) Y[(x / DV) * DY + DK + (x % DV)] = w.dUn[ci * C * DV + x];
    for (int r = tid; r < C; r += NT) {
        bs[r] = r < L ? to_f(io.beta[g.row(b, t0 + r, h)]) : 0.f;
        dbs[r] = 0.f;
    }
    __syncthreads();
    // M_ri = sum_c k_rc k_ic e^{g_rc - g_ic}  (i < r)
    for (int r = warp; r < C; r += NT / 32) {
        for (int i = 0; i < C; ++i) {
            float m = 0.f;
            if (i < r) {
                if (kda) {
                    for (int c = lane; c < DK; c += 32) m += ks[r * DK + c] * ks[i * DK + c] * __expf(gs[r * DK + c] - gs[i * DK + c]);
                } else {
                    for (int c = lane; c < DK; c += 32) m += ks[r * DK + c] * ks[i * DK + c];
                }
                m = warp_sum(m);
                if (g.variant == VAR_GATED) m *= __expf(gs[r * DK] - gs[i * DK]);
            }
            if (lane == 0) M[r * C + i] = m;
        }
    }
    __syncthreads();
    // back substitution: Y_i -= sum_{r>i} beta_r M_ri Y_r, i descending
    for (int x = tid; x < DY; x += NT) {
        for (int i = C - 2; i >= 0; --i) {
            float acc = Y[i * DY + x];
            for (int r = i + 1; r < C; ++r) acc -= bs[r] * M[r * C + i] * Y[r * DY + x];
            Y[i * DY + x] = acc;
        }
    }
    __syncthreads();
    // dA = -strict_tril([dB_k | dB_v] [W | U~]^T), dM = diag(beta) dA, dbeta (A part), and
    // dP = tril(dO U^T).  At C = 64: two 64 x 64 products, tiled through shared memory (the
    // dM | dP region, written only at the end) in steps of K; thread t owns rows 4 (t / 16) ..
    // + 3 and columns 4 (t % 16) .. + 3 of both results.  Smaller chunks: one warp per row.
    if (C != 64) {
        const float *Wg = w.W + ci * C * DK, *Ug = w.Ut + ci * C * DV, *Un = w.Un + ci * C * DV;
        for (int r = warp; r < C; r += NT / 32) {
            float db = 0.f;
            for (int i = 0; i < C; ++i) {
                float da = 0.f, dp = 0.f;
                if (i < r) {
                    for (int c = lane; c < DK; c += 32) da += Y[r * DY + c] * Wg[i * DK + c];
                    for (int j = lane; j < DV; j += 32) da += Y[r * DY + DK + j] * Ug[i * DV + j];
                    da = -warp_sum(da);
                    db += da * M[r * C + i];
                }
                if (i <= r && r < L && io.dout) {
                    const size_t row = g.row(b, t0 + r, h);
                    for (int j = lane; j < DV; j += 32) dp += to_f(io.dout[row * DV + j]) * Un[i * DV + j];
                    dp = warp_sum(dp);
                }
                if (lane == 0) {
                    dM[r * C + i] = bs[r] * da;
                    dP[r * C + i] = dp;
                }
            }
            if (lane == 0) dbs[r] += db;
        }
    } else {
        static_assert(NT == 256, "4 x 4 blocks of a 64 x 64 result");
        const float *Wg = w.W + ci * C * DK, *Ug = w.Ut + ci * C * DV, *Un = w.Un + ci * C * DV;
        float *stg = dM;  // 2 C C floats of staging
        const int r0 = 4 * (tid >> 4), i0 = 4 * (tid & 15);
        float da[4][4] = {}, dp[4][4] = {};
        // [dB_k | dB_v] (Y, already in shared memory) times [W | U~]^T, K = dk + dv in steps of 64
        constexpr int LD = 65;  // padded row stride of a staged 64 x 64 tile
        for (int k0 = 0; k0 < DY; k0 += 64) {
            __syncthreads();
            const float *src = k0 < DK ? Wg + k0 : Ug + (k0 - DK);
            const int ld = k0 < DK ? DK : DV;
            for (int x = tid; x < 64 * 64; x += NT) stg[(x >> 6) * LD + (x & 63)] = src[(x >> 6) * ld + (x & 63)];
            __syncthreads();
#pragma unroll 4
            for (int kk = 0; kk < 64; ++kk) {
                float av[4], bv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    av[u] = Y[(r0 + u) * DY + k0 + kk];
                    bv[u] = stg[(i0 + u) * LD + kk];
                }
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int v2 = 0; v2 < 4; ++v2) da[u][v2] += av[u] * bv[v2];
            }
        }
        // dO U^T, K = dv in steps of 32 (dO rows past T and a missing dO are zero)
        constexpr int LD2 = 33;
        for (int k0 = 0; k0 < DV && io.dout; k0 += 32) {
            __syncthreads();
            float *so = stg, *su = stg + 64 * LD2;
            for (int x = tid; x < 64 * 32; x += NT) {
                const int r = x >> 5, j = x & 31;
                so[r * LD2 + j] = r < L ? to_f(io.dout[g.row(b, t0 + r, h) * DV + k0 + j]) : 0.f;
                su[r * LD2 + j] = Un[r * DV + k0 + j];
            }
            __syncthreads();
#pragma unroll 4
            for (int kk = 0; kk < 32; ++kk) {
                float av[4], bv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    av[u] = so[(r0 + u) * LD2 + kk];
                    bv[u] = su[(i0 + u) * LD2 + kk];
                }
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int v2 = 0; v2 < 4; ++v2) dp[u][v2] += av[u] * bv[v2];
            }
        }
        __syncthreads();  // the staging region becomes dM | dP
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int r = r0 + u;
            float db = 0.f;
#pragma unroll
            for (int v2 = 0; v2 < 4; ++v2) {
                const int i = i0 + v2;
                const float a2 = i < r ? -da[u][v2] : 0.f;
                db += a2 * M[r * C + i];
                dM[r * C + i] = bs[r] * a2;
                dP[r * C + i] = i <= r ? dp[u][v2] : 0.f;
            }
            // the 16 threads of row block r0 / 4 are lanes 0-15 or 16-31 of one warp
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) db += __shfl_xor_sync(0xffffffffu, db, o);
            if ((tid & 15) == 0) dbs[r] += db;
        }
    }
    __syncthreads();
    if (!kda) {
        // scalar gates: fold the pair factor e^{g_r - g_i} (<= 1) into dM and dP once
        for (int x = tid; x < C * C; x += NT) {
            const int r = x / C, i = x % C;
            if (i <= r) {
                const float e = (g.variant == VAR_GATED) ? __expf(gs[r * DK] - gs[i * DK]) : 1.f;
                dM[x] *= e;
                dP[x] *= e;
            }
        }
        __syncthreads();
    }
    // per (r, c) gradients; dg_rc overwrites Y[r][c] (dB_k) -- each entry touched by one thread
    {
        const float *Qd = w.Qd + ci * C * DK, *Tm = w.Tm + ci * C * DK;
        for (int r = warp; r < C; r += NT / 32) {
            float dbk = 0.f;
            const size_t row = g.row(b, t0 + min(r, L - 1), h);
            for (int c = lane; c < DK; c += 32) {
                const float grc = gs[r * DK + c], gam = __expf(grc), kv = ks[r * DK + c], qv = qs[r * DK + c];
                const float gL = gs[(C - 1) * DK + c];
                float X = 0.f, Yv = 0.f, Z = 0.f;
                if (kda) {
                    for (int i = 0; i <= r; ++i) {
                        const float e = __expf(grc - gs[i * DK + c]) * ks[i * DK + c];
                        X += dP[r * C + i] * e;
                        Yv += dM[r * C + i] * e;  // dM[r][r] == 0
                    }
                    for (int rr = r; rr < C; ++rr) {
                        const float e = __expf(gs[rr * DK + c] - grc);
                        Z += (dM[rr * C + r] * ks[rr * DK + c] + dP[rr * C + r] * qs[rr * DK + c]) * e;
                    }
                } else {
                    for (int i = 0; i <= r; ++i) {
                        const float kic = ks[i * DK + c];
                        X += dP[r * C + i] * kic;
                        Yv += dM[r * C + i] * kic;
                    }
                    for (int rr = r; rr < C; ++rr) Z += dM[rr * C + r] * ks[rr * DK + c] + dP[rr * C + r] * qs[rr * DK + c];
                }
                const float qd = Qd[r * DK + c], tm = Tm[r * DK + c], dBk = Y[r * DY + c];
                const float eb = __expf(gL - grc);
                const float dq = gam * qd + X;
                const float dk = Yv + Z + bs[r] * gam * dBk + eb * tm;
                const float dg = qv * (gam * qd + X) + kv * (Yv - Z) + bs[r] * gam * kv * dBk - kv * eb * tm;
                dbk += gam * kv * dBk;
                Y[r * DY + c] = dg;
                if (r < L) {
                    io.dq[row * DK + c] = from_f<TI>(dq);
                    io.dk[row * DK + c] = from_f<TI>(dk);
                }
            }
            float dbv = 0.f;
            for (int j = lane; j < DV; j += 32) {
                const float dBv = Y[r * DY + DK + j];
                if (r < L) {
                    dbv += dBv * to_f(io.v[row * DV + j]);
                    io.dv[row * DV + j] = from_f<TI>(bs[r] * dBv);
                }
            }
            const float s = warp_sum(dbk + dbv);
            if (lane == 0) dbs[r] += s;
        }
    }
    __syncthreads();
    if (g.variant == VAR_DELTANET) {
        for (int r = tid; r < L; r += NT) io.dbeta[g.row(b, t0 + r, h)] = from_f<TI>(dbs[r]);
        return;
    }
    // dg_C: Kbar . Tm summed over rows, and gamma_C rowsum(S .* dS+); added to the last row
    {
        const float *Tm = w.Tm + ci * C * DK;
        for (int c = tid; c < DK; c += NT) {
            const float gL = gs[(C - 1) * DK + c];
            float acc = __expf(gL) * w.RS[ci * DK + c];
            for (int r = 0; r < C; ++r) acc += ks[r * DK + c] * __expf(gL - gs[r * DK + c]) * Tm[r * DK + c];
            Y[(C - 1) * DY + c] += acc;
        }
    }
    __syncthreads();
    if (kda) {
        for (int c = tid; c < DK; c += NT) {
            float run = 0.f;
            for (int r = C - 1; r >= 0; --r) {
                run += Y[r * DY + c];
                if (r < L) io.dalpha[g.row(b, t0 + r, h) * DK + c] = from_f<TI>(run);
            }
        }
    } else {
        for (int r = warp; r < C; r += NT / 32) {
            float s = 0.f;
            for (int c = lane; c < DK; c += 32) s += Y[r * DY + c];
            s = warp_sum(s);
            if (lane == 0) red[r] = s;
        }
        __syncthreads();
        if (tid == 0) {
            float run = 0.f;
            for (int r = C - 1; r >= 0; --r) {
                run += red[r];
                if (r < L) io.dalpha[g.row(b, t0 + r, h)] = from_f<TI>(run);
            }
        }
    }
    for (int r = tid; r < L; r += NT) io.dbeta[g.row(b, t0 + r, h)] = from_f<TI>(dbs[r]);
}

// ---------------------------------------------------------------------------------------------
// The same gradients at C = 64, with every per-(row, channel) sum written as a matrix product.
// KDA's pair factor is split at a per-channel midpoint m_c of the chunk's gates,
//   e^{g_rc - g_ic} = e^{g_rc - m_c} e^{m_c - g_ic},
// so that with Kp = k e^{g - m}, Km = k e^{m - g}, Qp = q e^{g - m}:
//   M  = strict_tril(Kp Km^T)
//   X  = e^{g - m} .* (dP Km),   Yv = e^{g - m} .* (dM Km)
//   Z  = e^{m - g} .* (dM^T Kp + dP^T Qp)
// It serves a chunk only when every channel's gates there span at most RANGE_MAX, so that every
// factor lies within e^{+-RANGE_MAX/2} and each product equals the direct sum up to rounding.
// The scalar gates fold their pair factor into M, dM and dP instead (Kp = Km = k, Qp = q).  The
// back substitution through (I+A)^T runs right-looking with one column of [dW | dU] in registers.
// smem: Kp, Km, Qp [64][dk]; Y [64][dk+dv]; M, dM, dP [64][LDC]; bs, dbs, red, grow [64]; gm [dk]
static constexpr int LDC = 68;             // padded row stride of the 64 x 64 matrices
static constexpr float RANGE_MAX = 120.f;  // widest in-chunk gate span of a channel (nats)

__host__ __device__ constexpr int tiled_gm_offset(int dk, int dv) {
    return 3 * 64 * dk + 64 * (dk + dv) + 3 * 64 * LDC + 4 * 64;
}
__device__ __forceinline__ float clamp_half_range(float x) {
    return fminf(fmaxf(x, -0.5f * RANGE_MAX), 0.5f * RANGE_MAX);
}

// acc[u][v] += sum_{k < K1 + K2} A[(r0 + u) lda + k] B(k)[i0 + v]: one thread's 4 x 4 block of a
// 64 x 64 product whose K columns come from B1 (ld1, K1 columns) and then B2 (ld2, K2 columns).
// B passes through stg (64 x 65 floats) 64 columns at a time, the next block held in registers
// while the current one is multiplied.  K1 and K2 are multiples of 64.  The first block of B is
// read before the first barrier: a B in shared memory must be complete when nt64 is called.
// The caller synchronises before stg is written again.
__device__ __forceinline__ void nt64(const float *A, int lda, const float *B1, int ld1, int K1, const float *B2,
                                     int ld2, int K2, float *stg, int r0, int i0, float (&acc)[4][4]) {
    constexpr int LD = 65, PER = 64 * 64 / NT;
    const int K = K1 + K2;
    float nxt[PER];
    auto fetch = [&](int k0) {
        const float *B = k0 < K1 ? B1 + k0 : B2 + (k0 - K1);
        const int ldb = k0 < K1 ? ld1 : ld2;
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            const int x = threadIdx.x + e * NT;
            nxt[e] = B[(size_t)(x >> 6) * ldb + (x & 63)];
        }
    };
    fetch(0);
    for (int k0 = 0; k0 < K; k0 += 64) {
        __syncthreads();
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            const int x = threadIdx.x + e * NT;
            stg[(x >> 6) * LD + (x & 63)] = nxt[e];
        }
        __syncthreads();
        if (k0 + 64 < K) fetch(k0 + 64);
#pragma unroll 4
        for (int kk = 0; kk < 64; ++kk) {
            float av[4], bv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                av[u] = A[(r0 + u) * lda + k0 + kk];
                bv[u] = stg[(i0 + u) * LD + kk];
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 4; ++v) acc[u][v] += av[u] * bv[v];
        }
    }
}

template <int N> __device__ __forceinline__ void ld4s(float (&d)[N], const float *p) {
#pragma unroll
    for (int v = 0; v < N; v += 4) {
        const float4 t = *reinterpret_cast<const float4 *>(p + v);
        d[v] = t.x; d[v + 1] = t.y; d[v + 2] = t.z; d[v + 3] = t.w;
    }
}

template <typename TI, int DK, int DV>
__device__ __forceinline__ void intra_tiled(const Geo &g, const IO<TI> &io, const SimtWs &w) {
    constexpr int C = 64, DY = DK + DV, CW = DK / 16;
    static_assert(NT == 256, "16 x 16 thread blocks over the 64 x 64 products");
    const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int t0 = n * C, L = min(C, g.T - t0);
    extern __shared__ float sm[];
    float *Kp = sm, *Km = Kp + C * DK, *Qp = Km + C * DK, *Y = Qp + C * DK;
    float *M = Y + C * DY, *dM = M + C * LDC, *dP = dM + C * LDC;
    float *bs = dP + C * LDC, *dbs = bs + C, *red = dbs + C, *grow = red + C, *gm = grow + C;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool kda = g.variant == VAR_KDA, gated = g.variant == VAR_GATED;
    const size_t ci = g.chunk(b, h, n);
    const float *Gg = w.G + ci * C * DK;

    // loads in batches of 8 per thread, all issued before any is used
#pragma unroll
    for (int e0 = 0; e0 < C * DK / NT; e0 += 8) {
        float kv[8], qv[8], gv[8], dw[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int x = tid + (e0 + e) * NT, r = x / DK, c = x % DK;
            const size_t row = g.row(b, t0 + min(r, L - 1), h);
            kv[e] = to_f(io.k[row * DK + c]);
            qv[e] = to_f(io.q[row * DK + c]);
            gv[e] = Gg[x];
            dw[e] = w.dWm[ci * C * DK + x];
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int x = tid + (e0 + e) * NT, r = x / DK, c = x % DK;
            const float k1 = r < L ? kv[e] : 0.f, q1 = r < L ? qv[e] : 0.f;
            float ep = 1.f, em = 1.f;
            if (kda) {
                const float a = clamp_half_range(gv[e] - gm[c]);
                ep = __expf(a);
                em = __expf(-a);
            }
            Kp[x] = k1 * ep; Km[x] = k1 * em; Qp[x] = q1 * ep;
            Y[r * DY + c] = dw[e];
        }
    }
#pragma unroll
    for (int e0 = 0; e0 < C * DV / NT; e0 += 8) {
        float du[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) du[e] = w.dUn[ci * C * DV + tid + (e0 + e) * NT];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int x = tid + (e0 + e) * NT;
            Y[(x / DV) * DY + DK + (x % DV)] = du[e];
        }
    }
    for (int r = tid; r < C; r += NT) {
        bs[r] = r < L ? to_f(io.beta[g.row(b, t0 + r, h)]) : 0.f;
        dbs[r] = 0.f;
        grow[r] = Gg[r * DK];
    }
    // 4 x 4 blocks of the 64 x 64 products: rows r0.., columns i0..
    const int r0 = 4 * (tid >> 4), i0 = 4 * (tid & 15);
    {
        float acc[4][4] = {};
        // nt64 reads its first block of B (here Km, written above by other threads) before its
        // first barrier, so the loads are published here
        __syncthreads();
        nt64(Kp, DK, Km, DK, DK, nullptr, 0, 0, dM, r0, i0, acc);
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const int r = r0 + u, i = i0 + v;
                float m = 0.f;
                if (i < r) m = gated ? acc[u][v] * __expf(grow[r] - grow[i]) : acc[u][v];
                M[r * LDC + i] = m;
            }
    }
    __syncthreads();
    // [dB_k | dB_v]_i = Y_i - sum_{r > i} beta_r M_ri [dB]_r: once row r is final it updates every
    // row above it, so the 63 steps each carry up to 63 independent updates
    if (tid < DY) {
        float y[C];
#pragma unroll
        for (int r = 0; r < C; ++r) y[r] = Y[r * DY + tid];
#pragma unroll
        for (int r = C - 1; r >= 1; --r) {
            const float t = bs[r] * y[r];
#pragma unroll
            for (int i = 0; i < r; i += 4) {
                const float4 m4 = *reinterpret_cast<const float4 *>(M + r * LDC + i);
                y[i] -= m4.x * t;
                if (i + 1 < r) y[i + 1] -= m4.y * t;
                if (i + 2 < r) y[i + 2] -= m4.z * t;
                if (i + 3 < r) y[i + 3] -= m4.w * t;
            }
        }
#pragma unroll
        for (int r = 0; r < C; ++r) Y[r * DY + tid] = y[r];
    }
    // dA = -strict_tril([dB_k | dB_v] [W | U~]^T), dM = diag(beta) dA, the A part of dbeta, and
    // dP = tril(dO U^T)
    {
        const float *Wg = w.W + ci * C * DK, *Ug = w.Ut + ci * C * DV, *Un = w.Un + ci * C * DV;
        float da[4][4] = {}, dp[4][4] = {};
        nt64(Y, DY, Wg, DK, DK, Ug, DV, DV, dM, r0, i0, da);
        constexpr int LD2 = 33, PER2 = 64 * 32 / NT;
        float *so = dM, *su = dM + 64 * LD2;
        float no[PER2], nu[PER2];
        auto fetch2 = [&](int k0) {
#pragma unroll
            for (int e = 0; e < PER2; ++e) {
                const int x = tid + e * NT, r = x >> 5, j = x & 31;
                no[e] = to_f(io.dout[g.row(b, t0 + min(r, L - 1), h) * DV + k0 + j]);
                nu[e] = Un[r * DV + k0 + j];
            }
        };
        if (io.dout) fetch2(0);
        for (int k0 = 0; k0 < DV && io.dout; k0 += 32) {
            __syncthreads();
#pragma unroll
            for (int e = 0; e < PER2; ++e) {
                const int x = tid + e * NT, r = x >> 5, j = x & 31;
                so[r * LD2 + j] = r < L ? no[e] : 0.f;
                su[r * LD2 + j] = nu[e];
            }
            __syncthreads();
            if (k0 + 32 < DV) fetch2(k0 + 32);
#pragma unroll 4
            for (int kk = 0; kk < 32; ++kk) {
                float av[4], bv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    av[u] = so[(r0 + u) * LD2 + kk];
                    bv[u] = su[(i0 + u) * LD2 + kk];
                }
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int v = 0; v < 4; ++v) dp[u][v] += av[u] * bv[v];
            }
        }
        __syncthreads();  // the staging region becomes dM | dP
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int r = r0 + u;
            float db = 0.f;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const int i = i0 + v;
                const float a2 = i < r ? -da[u][v] : 0.f;
                db += a2 * M[r * LDC + i];
                const float e = (gated && i <= r) ? __expf(grow[r] - grow[i]) : 1.f;
                dM[r * LDC + i] = bs[r] * a2 * e;
                dP[r * LDC + i] = i <= r ? dp[u][v] * e : 0.f;
            }
            // the 16 threads of one row block are lanes 0-15 or 16-31 of a warp
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) db += __shfl_xor_sync(0xffffffffu, db, o);
            if ((tid & 15) == 0) dbs[r] += db;
        }
    }
    __syncthreads();
    // dv and the v part of dbeta, one warp per row
#pragma unroll
    for (int r = warp; r < C; r += NT / 32) {
        float dbv = 0.f;
        if (r < L) {
            const size_t row = g.row(b, t0 + r, h);
            float vv[DV / 32];
#pragma unroll
            for (int e = 0; e < DV / 32; ++e) vv[e] = to_f(io.v[row * DV + lane + 32 * e]);
#pragma unroll
            for (int e = 0; e < DV / 32; ++e) {
                const float dBv = Y[r * DY + DK + lane + 32 * e];
                dbv += dBv * vv[e];
                io.dv[row * DV + lane + 32 * e] = from_f<TI>(bs[r] * dBv);
            }
        }
        dbv = warp_sum(dbv);
        if (lane == 0) dbs[r] += dbv;
    }
    // [64][dk] products: warp w owns the 8 rows of group rg (the two halves of the warp 4 each) and
    // all dk columns, CW per lane.  dP and dM are lower triangular, so the first products stop at
    // the group's last row and the transposed ones start at its first; warps w and w + 4 share a
    // scheduler and get groups rg and 7 - rg, the same number of steps between them.
    const int rg = warp < 4 ? warp : 11 - warp;
    const int rb = 2 * rg + (lane >> 4), q0 = 4 * rb, c0 = CW * (lane & 15);
    float *part = M;  // [16][dk] row-block sums of k e^{g_C - g} Tm (M is not read again)
    const float *Qd = w.Qd + ci * C * DK, *Tm = w.Tm + ci * C * DK;
    {
        float X[4][CW], V[4][CW];
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int v = 0; v < CW; ++v) X[u][v] = V[u][v] = 0.f;
        const int iend = 8 * rg + 8;
        for (int i = 0; i < iend; ++i) {
            float ap[4], am[4], bk[CW];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                ap[u] = dP[(q0 + u) * LDC + i];
                am[u] = dM[(q0 + u) * LDC + i];
            }
            ld4s(bk, Km + i * DK + c0);
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < CW; ++v) {
                    X[u][v] += ap[u] * bk[v];
                    V[u][v] += am[u] * bk[v];
                }
        }
        __syncthreads();  // Km and M are overwritten below
        float dgc[CW], gl[CW];
        ld4s(gl, Gg + (C - 1) * DK + c0);
#pragma unroll
        for (int v = 0; v < CW; ++v) dgc[v] = 0.f;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int r = q0 + u;
            const bool live = r < L;
            const size_t row = g.row(b, t0 + min(r, L - 1), h);
            float gr[CW], qdv[CW], tmv[CW], kr[CW], qr[CW];
            ld4s(gr, Gg + r * DK + c0);
            ld4s(qdv, Qd + r * DK + c0);
            ld4s(tmv, Tm + r * DK + c0);
#pragma unroll
            for (int v = 0; v < CW; ++v) {
                kr[v] = to_f(io.k[row * DK + c0 + v]);
                qr[v] = to_f(io.q[row * DK + c0 + v]);
            }
            float dbk = 0.f;
#pragma unroll
            for (int v = 0; v < CW; ++v) {
                const int c = c0 + v;
                const float grc = gr[v], gam = __expf(grc), eb = __expf(gl[v] - grc);
                const float kv = live ? kr[v] : 0.f, qv = live ? qr[v] : 0.f;
                const float f = kda ? __expf(clamp_half_range(grc - gm[c])) : 1.f;
                const float xs = X[u][v] * f, ys = V[u][v] * f;
                const float dBk = Y[r * DY + c], et = eb * tmv[v];
                const float dq = gam * qdv[v] + xs, sb = bs[r] * gam * dBk;
                Km[r * DK + c] = ys + sb + et;                  // dk but for its Z term
                Y[r * DY + c] = qv * dq + kv * (ys + sb - et);  // dg but for its -k Z term
                dbk += kv * gam * dBk;
                dgc[v] += kv * et;
                if (live) io.dq[row * DK + c] = from_f<TI>(dq);
            }
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) dbk += __shfl_xor_sync(0xffffffffu, dbk, o);
            if ((lane & 15) == 0) dbs[r] += dbk;
        }
#pragma unroll
        for (int v = 0; v < CW; ++v) part[rb * DK + c0 + v] = dgc[v];
    }
    {
        float Z[4][CW];
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int v = 0; v < CW; ++v) Z[u][v] = 0.f;
        for (int r2 = 8 * rg; r2 < C; ++r2) {
            float am[4], ap[4], bk[CW], bq[CW];
            ld4s(am, dM + r2 * LDC + q0);
            ld4s(ap, dP + r2 * LDC + q0);
            ld4s(bk, Kp + r2 * DK + c0);
            ld4s(bq, Qp + r2 * DK + c0);
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < CW; ++v) Z[u][v] += am[u] * bk[v] + ap[u] * bq[v];
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int r = q0 + u;
            const bool live = r < L;
            const size_t row = g.row(b, t0 + min(r, L - 1), h);
            float gr[CW], kr[CW];
            ld4s(gr, Gg + r * DK + c0);
#pragma unroll
            for (int v = 0; v < CW; ++v) kr[v] = to_f(io.k[row * DK + c0 + v]);
#pragma unroll
            for (int v = 0; v < CW; ++v) {
                const int c = c0 + v;
                const float f = kda ? __expf(clamp_half_range(gm[c] - gr[v])) : 1.f;
                const float z = Z[u][v] * f;
                const float kv = live ? kr[v] : 0.f;
                if (live) io.dk[row * DK + c] = from_f<TI>(Km[r * DK + c] + z);
                Y[r * DY + c] -= kv * z;
            }
        }
    }
    __syncthreads();
    if (g.variant == VAR_DELTANET) {
        for (int r = tid; r < L; r += NT) io.dbeta[g.row(b, t0 + r, h)] = from_f<TI>(dbs[r]);
        return;
    }
    // dg_C: the K-bar . Tm sums and gamma_C rowsum(S .* dS+), added to the last row
    for (int c = tid; c < DK; c += NT) {
        float acc = __expf(Gg[(C - 1) * DK + c]) * w.RS[ci * DK + c];
#pragma unroll
        for (int p = 0; p < 16; ++p) acc += part[p * DK + c];
        Y[(C - 1) * DY + c] += acc;
    }
    __syncthreads();
    if (kda) {
        for (int c = tid; c < DK; c += NT) {
            float run = 0.f;
            for (int r = C - 1; r >= 0; --r) {
                run += Y[r * DY + c];
                if (r < L) io.dalpha[g.row(b, t0 + r, h) * DK + c] = from_f<TI>(run);
            }
        }
    } else {
        for (int r = warp; r < C; r += NT / 32) {
            float s = 0.f;
            for (int c = lane; c < DK; c += 32) s += Y[r * DY + c];
            s = warp_sum(s);
            if (lane == 0) red[r] = s;
        }
        __syncthreads();
        if (tid == 0) {
            float run = 0.f;
            for (int r = C - 1; r >= 0; --r) {
                run += red[r];
                if (r < L) io.dalpha[g.row(b, t0 + r, h)] = from_f<TI>(run);
            }
        }
    }
    for (int r = tid; r < L; r += NT) io.dbeta[g.row(b, t0 + r, h)] = from_f<TI>(dbs[r]);
}

// One chunk per CTA.  At C = 64 a KDA chunk first finds each channel's midpoint and span; the
// factorised form takes every chunk it accepts, the direct form the rest.
template <typename TI>
__global__ void __launch_bounds__(NT) k_bwd_intra(Geo g, IO<TI> io, SimtWs w) {
    if (w.only && !w.only[g.chunk(blockIdx.z, blockIdx.y, blockIdx.x)]) return;  // uniform over the CTA
    if (g.C == 64) {
        int wide = 0;
        if (g.variant == VAR_KDA) {
            extern __shared__ float sm[];
            float *gm = sm + tiled_gm_offset(g.dk, g.dv);
            const int n = blockIdx.x, L = min(64, g.T - n * 64);
            const float *Gg = w.G + g.chunk(blockIdx.z, blockIdx.y, n) * 64 * g.dk;
            for (int c = threadIdx.x; c < g.dk; c += NT) {
                float hi = Gg[c], lo = Gg[c];
#pragma unroll 16
                for (int r = 1; r < L; ++r) {
                    const float v = Gg[r * g.dk + c];
                    hi = fmaxf(hi, v);
                    lo = fminf(lo, v);
                }
                gm[c] = 0.5f * (hi + lo);
                if (!(hi - lo <= RANGE_MAX)) wide = 1;
            }
        }
        if (!__syncthreads_or(wide)) {
            if (g.dk == 128) {
                if (g.dv == 128) intra_tiled<TI, 128, 128>(g, io, w);
                else intra_tiled<TI, 128, 64>(g, io, w);
            } else {
                if (g.dv == 128) intra_tiled<TI, 64, 128>(g, io, w);
                else intra_tiled<TI, 64, 64>(g, io, w);
            }
            return;
        }
    }
    intra_direct<TI>(g, io, w);
}

// ---------------------------------------------------------------------------------------------
// host side
static size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t simt_ws_bytes(const Geo &g, bool bwd) {
    const size_t nc = (size_t)g.B * g.H * g.N, C = g.C, DK = g.dk, DV = g.dv;
    size_t s = 0;
    s += al256(nc * C * DK * 4);   // W
    s += al256(nc * C * DV * 4);   // Ut
    s += al256(nc * C * DK * 4);   // G
    s += al256(nc * C * C * 4);    // P
    s += al256(nc * DK * DV * 4);  // Sn
    s += al256(nc * C * DV * 4);   // Un
    if (bwd) {
        s += al256(nc * DK * DV * 4);     // dSn
        s += al256(nc * C * DV * 4);      // dUn
        s += 3 * al256(nc * C * DK * 4);  // Qd dWm Tm
        s += al256(nc * DK * 4);          // RS
    }
    return s;
}

SimtWs simt_ws_carve(const Geo &g, bool bwd, void *base) {
    const size_t nc = (size_t)g.B * g.H * g.N, C = g.C, DK = g.dk, DV = g.dv;
    char *p = (char *)base;
    auto take = [&](size_t bytes) { float *r = (float *)p; p += al256(bytes); return r; };
    SimtWs w = {};
    w.W = take(nc * C * DK * 4);
    w.Ut = take(nc * C * DV * 4);
    w.G = take(nc * C * DK * 4);
    w.P = take(nc * C * C * 4);
    w.Sn = take(nc * DK * DV * 4);
    w.Un = take(nc * C * DV * 4);
    if (bwd) {
        w.dSn = take(nc * DK * DV * 4);
        w.dUn = take(nc * C * DV * 4);
        w.Qd = take(nc * C * DK * 4);
        w.dWm = take(nc * C * DK * 4);
        w.Tm = take(nc * C * DK * 4);
        w.RS = take(nc * DK * 4);
    }
    return w;
}

template <typename K> static cudaError_t prep_attr(K kern, size_t smem) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
}

#define DR_TRY(x)                                \
    do {                                         \
        cudaError_t e__ = (x);                   \
        if (e__ != cudaSuccess) return e__;      \
    } while (0)

const char *const SIMT_FWD_KERNELS[3] = {"k_prep", "k_scan", "k_out"};
const char *const SIMT_BWD_KERNELS[5] = {"k_prep", "k_scan", "k_scan_bwd", "k_bwd_state", "k_bwd_intra"};

template <typename TI>
static cudaError_t forward_chain(const Geo &g, const IO<TI> &io, const SimtWs &w, const float *S0, float *ST,
                                 int write_u, cudaStream_t s, Rec &rec) {
    const size_t C = g.C, DK = g.dk, DV = g.dv;
    const dim3 gc(g.N, g.H, g.B), gs(g.dv / JB, g.H, g.B);
    const size_t sm_prep = 4 * (3 * C * DK + C * DV + 2 * C * C + C);
    DR_TRY(prep_attr(k_prep<TI>, sm_prep));
    const size_t sm_scan = 4 * (DK * JB + 2 * C * DK + C * JB + DK);
    DR_TRY(prep_attr(k_scan<TI>, sm_scan));
    rec.mark(s);
    k_prep<TI><<<gc, NT, sm_prep, s>>>(g, io, w);
    DR_TRY(cudaGetLastError());
    rec.mark(s);
    k_scan<TI><<<gs, NT, sm_scan, s>>>(g, io, w, S0, ST, write_u);
    return cudaGetLastError();
}

template <typename TI>
static cudaError_t fwd_t(const Geo &g, const Tensors &t, const SimtWs &w, cudaStream_t s, Rec &rec) {
    const IO<TI> io = io_of<TI>(t);
    const size_t C = g.C, DK = g.dk;
    const size_t sm_out = 4 * (C * DK + C * C + DK * JB + C * JB);
    DR_TRY(prep_attr(k_out<TI>, sm_out));
    DR_TRY(forward_chain<TI>(g, io, w, t.S0, t.S_T, t.u != nullptr, s, rec));
    rec.mark(s);
    k_out<TI><<<dim3(g.N, g.H, g.B), NT, sm_out, s>>>(g, io, w);
    return cudaGetLastError();
}

// from = 0: everything; 1: the forward's W, U~, G, P, S_n, U are in w already; 2: so are the
// reverse chain's dS_{n+1} and dU (and dS0 is written); 3: so are the state products Qd, dWm,
// Tm, RS (only k_bwd_intra runs)
template <typename TI>
static cudaError_t bwd_t(const Geo &g, const Tensors &t, const SimtWs &w, int from, cudaStream_t s, Rec &rec) {
    const IO<TI> io = io_of<TI>(t);
    const size_t C = g.C, DK = g.dk, DV = g.dv;
    const dim3 gc(g.N, g.H, g.B), gs(g.dv / JB, g.H, g.B);
    const size_t sm_sb = 4 * (DK * JB + 3 * C * DK + C * C + 2 * C * JB + DK);
    const size_t sm_st = C == 64 ? 2 * 4 * (2 * DK + 3 * C) * (JB + 1)
                                 : 4 * (3 * C * DK + 2 * DK * (JB + 1) + 3 * C * JB + DK);
    size_t sm_in = 4 * (3 * C * DK + C * (DK + DV) + 3 * C * C + 3 * C);
    const size_t sm_tiled = 4 * ((size_t)tiled_gm_offset((int)DK, (int)DV) + DK);
    if (C == 64 && sm_tiled > sm_in) sm_in = sm_tiled;
    DR_TRY(prep_attr(k_scan_bwd<TI>, sm_sb));
    DR_TRY(prep_attr(k_bwd_state<TI>, sm_st));
    DR_TRY(prep_attr(k_bwd_intra<TI>, sm_in));
    if (from == 0) DR_TRY(forward_chain<TI>(g, io, w, t.S0, nullptr, 0, s, rec));
    if (from < 2) {
        rec.mark(s);
        k_scan_bwd<TI><<<gs, NT, sm_sb, s>>>(g, io, w, t.dS_T, t.dS0);
        DR_TRY(cudaGetLastError());
    }
    if (from < 3) {
        rec.mark(s);
        k_bwd_state<TI><<<gc, NT, sm_st, s>>>(g, io, w);
        DR_TRY(cudaGetLastError());
    }
    rec.mark(s);
    k_bwd_intra<TI><<<gc, NT, sm_in, s>>>(g, io, w);
    return cudaGetLastError();
}

cudaError_t simt_fwd(const Geo &g, const Tensors &t, bool bf16, const SimtWs &w, cudaStream_t s, Rec &rec) {
    return bf16 ? fwd_t<__nv_bfloat16>(g, t, w, s, rec) : fwd_t<float>(g, t, w, s, rec);
}

cudaError_t simt_bwd(const Geo &g, const Tensors &t, bool bf16, const SimtWs &w, cudaStream_t s, Rec &rec) {
    return bf16 ? bwd_t<__nv_bfloat16>(g, t, w, 0, s, rec) : bwd_t<float>(g, t, w, 0, s, rec);
}

cudaError_t simt_bwd_grads(const Geo &g, const Tensors &t, bool bf16, const SimtWs &w, cudaStream_t s, Rec &rec) {
    return bf16 ? bwd_t<__nv_bfloat16>(g, t, w, 2, s, rec) : bwd_t<float>(g, t, w, 2, s, rec);
}

cudaError_t simt_bwd_intra(const Geo &g, const Tensors &t, bool bf16, const SimtWs &w, cudaStream_t s, Rec &rec) {
    return bf16 ? bwd_t<__nv_bfloat16>(g, t, w, 3, s, rec) : bwd_t<float>(g, t, w, 3, s, rec);
}

}  // namespace dr
