/*
 * delta_rule_oracle.c -- plain fp64 CPU oracle for the gated delta rule.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the independent checker for the CUDA
 * library in gated_delta_rule_107_b200/csrc.  It shares no code, header, table or
 * helper with that library, and the product path never calls it.  Only tests/,
 * __graft_entry__.smoke() and bench.py's cpu_baseline / reference legs use it.
 *
 * What it computes (all arithmetic in double precision):
 *
 *   "线性注意力架构演进与Kimi Delta Attention创新实践" (Kimi Delta Attention page),
 *   section 2.1, state-update equation:
 *       S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
 *       o_t = S_t^T q_t,           S in R^{dk x dv}.
 *   Variants ("线性注意力架构：机制、权衡与跨层路由" explainer, core method 1, and
 *   the ETH news article section 二):
 *       DeltaNet       alpha == 1
 *       Gated DeltaNet one scalar alpha per (token, head)
 *       KDA            one alpha per key channel (vector in (0,1)^dk)
 *   The gate is passed in log space (Kimi Delta Attention page, section 7.1:
 *   cumulative decay is accumulated by log-space addition).
 *
 *   Write value routed by CLVR (explainer, "4. 跨层路由 CLVR"; chatpaper abstract):
 *       S'_t = Diag(alpha_t) S_{t-1},  e_t = v_t - S'_t^T k_t,  u_t = beta_t e_t,
 *       S_t  = S'_t + k_t u_t^T.
 *   Expanding S'_t + k_t u_t^T gives exactly the section-2.1 equation, so this is
 *   the same recurrence written as "decay, predict, write the correction".
 *
 * Three entry points:
 *   oracle_fwd          token-by-token recurrence (the definition).
 *   oracle_bwd          reverse-mode adjoint of oracle_fwd for the loss
 *                       L = <dO,o> + <du,u> + <dS_T,S_T>; states are recomputed
 *                       from checkpoints taken every ORACLE_SEG steps.
 *   oracle_chunked_fwd  the chunkwise-parallel (UT / WY) form of the same map on
 *                       chunks of `chunk` tokens (Kimi Delta Attention page,
 *                       sections 6.1-6.2: chunked computation and the UT
 *                       transform), solving each chunk's (I + A) system by dense
 *                       Gaussian elimination.  Used only to pin the chunk algebra
 *                       against the token recurrence on small inputs.
 *
 * Layouts (row-major, contiguous):
 *   q, k        [B, T, H, dk]
 *   v, o, u     [B, T, H, dv]
 *   loga        [B, T, H]      (Gated DeltaNet)  or  [B, T, H, dk] (KDA);
 *               ignored (may be NULL) for DeltaNet
 *   beta        [B, T, H]
 *   S0, S_T     [B, H, dk, dv] (S0 == NULL means a zero initial state)
 * Any output pointer may be NULL (that output is skipped).
 * (b, h) pairs are independent; they are spread over `nthreads` POSIX threads
 * (0 = one per online core).
 * Return value: 0 on success, -1 on bad arguments, -2 on allocation failure.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORACLE_DELTANET 0
#define ORACLE_GATED 1
#define ORACLE_KDA 2
#define ORACLE_SEG 64 /* checkpoint spacing of the backward recompute */

typedef struct {
    /* forward inputs */
    const double *q, *k, *v, *loga, *beta, *S0;
    /* forward outputs */
    double *o, *u, *ST;
    /* backward inputs / outputs */
    const double *dO, *du, *dST;
    double *dq, *dk, *dv, *dloga, *dbeta, *dS0;
    int B, T, H, DK, DV, variant, chunk;
    /* work distribution */
    int next_unit;
    int failed;
    pthread_mutex_t lock;
} job_t;

/* ---- indexing helpers: element offsets of one (b, t, h) row ---- */
static size_t row_k(const job_t *J, int b, int t, int h) { return (((size_t)b * J->T + t) * J->H + h) * J->DK; }
static size_t row_v(const job_t *J, int b, int t, int h) { return (((size_t)b * J->T + t) * J->H + h) * J->DV; }
static size_t row_s(const job_t *J, int b, int t, int h) { return ((size_t)b * J->T + t) * J->H + h; }
static size_t state_off(const job_t *J, int b, int h) { return ((size_t)b * J->H + h) * J->DK * J->DV; }

/* alpha_t for channel c (the decay that Diag(alpha_t) applies to row c of S). */
static double gate(const job_t *J, int b, int t, int h, int c) {
    if (J->variant == ORACLE_DELTANET) return 1.0;
    if (J->variant == ORACLE_GATED) return exp(J->loga[row_s(J, b, t, h)]);
    return exp(J->loga[row_k(J, b, t, h) + c]);
}

/* log alpha_t for channel c. */
static double log_gate(const job_t *J, int b, int t, int h, int c) {
    if (J->variant == ORACLE_DELTANET) return 0.0;
    if (J->variant == ORACLE_GATED) return J->loga[row_s(J, b, t, h)];
    return J->loga[row_k(J, b, t, h) + c];
}

/*
 * One step of the recurrence on state S (dk x dv, row c = key channel).
 * On return S holds S_t; Sp (if non-NULL) holds S'_t = Diag(alpha_t) S_{t-1};
 * e and u hold the prediction error and the write value.
 */
static void step(const job_t *J, int b, int t, int h, double *S, double *Sp, double *e, double *u) {
    const int DK = J->DK, DV = J->DV;
    const double *kt = J->k + row_k(J, b, t, h);
    const double *vt = J->v + row_v(J, b, t, h);
    const double bt = J->beta[row_s(J, b, t, h)];
    /* S' = Diag(alpha) S */
    for (int c = 0; c < DK; ++c) {
        const double a = gate(J, b, t, h, c);
        for (int j = 0; j < DV; ++j) S[c * DV + j] *= a;
    }
    if (Sp) memcpy(Sp, S, sizeof(double) * DK * DV);
    /* e = v - S'^T k ;  u = beta e */
    for (int j = 0; j < DV; ++j) {
        double pred = 0.0;
        for (int c = 0; c < DK; ++c) pred += S[c * DV + j] * kt[c];
        e[j] = vt[j] - pred;
        u[j] = bt * e[j];
    }
    /* S = S' + k u^T */
    for (int c = 0; c < DK; ++c)
        for (int j = 0; j < DV; ++j) S[c * DV + j] += kt[c] * u[j];
}

static void load_initial_state(const job_t *J, int b, int h, double *S) {
    const size_t n = (size_t)J->DK * J->DV;
    if (J->S0) memcpy(S, J->S0 + state_off(J, b, h), sizeof(double) * n);
    else memset(S, 0, sizeof(double) * n);
}

/* ------------------------------------------------------------------------- */
/* forward: token-by-token                                                    */
/* ------------------------------------------------------------------------- */
static int fwd_unit(job_t *J, int b, int h) {
    const int DK = J->DK, DV = J->DV;
    double *S = malloc(sizeof(double) * DK * DV);
    double *e = malloc(sizeof(double) * DV);
    double *u = malloc(sizeof(double) * DV);
    if (!S || !e || !u) { free(S); free(e); free(u); return -2; }
    load_initial_state(J, b, h, S);
    for (int t = 0; t < J->T; ++t) {
        step(J, b, t, h, S, NULL, e, u);
        if (J->u) memcpy(J->u + row_v(J, b, t, h), u, sizeof(double) * DV);
        if (J->o) {
            /* o = S_t^T q */
            const double *qt = J->q + row_k(J, b, t, h);
            double *ot = J->o + row_v(J, b, t, h);
            for (int j = 0; j < DV; ++j) {
                double acc = 0.0;
                for (int c = 0; c < DK; ++c) acc += S[c * DV + j] * qt[c];
                ot[j] = acc;
            }
        }
    }
    if (J->ST) memcpy(J->ST + state_off(J, b, h), S, sizeof(double) * DK * DV);
    free(S); free(e); free(u);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* backward: reverse-mode adjoint of fwd_unit                                 */
/* ------------------------------------------------------------------------- */
/*
 * Loss L = <dO, o> + <du, u> + <dS_T, S_T>.  With G = dL/dS_t accumulated from
 * the end, one reverse step of  S'=Diag(a)S_{t-1}, e=v-S'^T k, u=beta e,
 * S_t = S' + k u^T, o = S_t^T q  is:
 *   G    += q dO^T                 dq = S_t dO
 *   dU    = du + G^T k             dv = beta dU,      dbeta = e . dU
 *   dk    = G u - beta S' dU
 *   dS'   = G - beta k dU^T
 *   dloga = rowsum(dS' .* S')  (per channel; summed over channels for Gated)
 *   G     = Diag(a) dS'            (= dL/dS_{t-1}; at t = 0 this is dS0)
 */
static int bwd_unit(job_t *J, int b, int h) {
    const int DK = J->DK, DV = J->DV, T = J->T;
    const size_t ns = (size_t)DK * DV;
    const int nseg = (T + ORACLE_SEG - 1) / ORACLE_SEG;
    int rc = 0;
    double *ckpt = malloc(sizeof(double) * ns * (size_t)(nseg > 0 ? nseg : 1)); /* S entering each segment */
    double *Sseg = malloc(sizeof(double) * ns * ORACLE_SEG);                 /* S_t inside a segment */
    double *Spseg = malloc(sizeof(double) * ns * ORACLE_SEG);                /* S'_t inside a segment */
    double *eseg = malloc(sizeof(double) * DV * ORACLE_SEG);
    double *useg = malloc(sizeof(double) * DV * ORACLE_SEG);
    double *S = malloc(sizeof(double) * ns);
    double *G = malloc(sizeof(double) * ns);
    double *dSp = malloc(sizeof(double) * ns);
    double *dU = malloc(sizeof(double) * DV);
    if (!ckpt || !Sseg || !Spseg || !eseg || !useg || !S || !G || !dSp || !dU) { rc = -2; goto done; }

    /* forward sweep, keeping the state at every segment start */
    load_initial_state(J, b, h, S);
    for (int t = 0; t < T; ++t) {
        if (t % ORACLE_SEG == 0) memcpy(ckpt + (size_t)(t / ORACLE_SEG) * ns, S, sizeof(double) * ns);
        step(J, b, t, h, S, NULL, eseg, useg);
    }

    if (J->dST) memcpy(G, J->dST + state_off(J, b, h), sizeof(double) * ns);
    else memset(G, 0, sizeof(double) * ns);

    for (int sg = nseg - 1; sg >= 0; --sg) {
        const int t0 = sg * ORACLE_SEG;
        const int t1 = (t0 + ORACLE_SEG < T) ? t0 + ORACLE_SEG : T;
        /* recompute the segment */
        memcpy(S, ckpt + (size_t)sg * ns, sizeof(double) * ns);
        for (int t = t0; t < t1; ++t) {
            const int i = t - t0;
            step(J, b, t, h, S, Spseg + (size_t)i * ns, eseg + (size_t)i * DV, useg + (size_t)i * DV);
            memcpy(Sseg + (size_t)i * ns, S, sizeof(double) * ns);
        }
        /* reverse through it */
        for (int t = t1 - 1; t >= t0; --t) {
            const int i = t - t0;
            const double *St = Sseg + (size_t)i * ns;
            const double *Sp = Spseg + (size_t)i * ns;
            const double *et = eseg + (size_t)i * DV;
            const double *ut = useg + (size_t)i * DV;
            const double *qt = J->q + row_k(J, b, t, h);
            const double *kt = J->k + row_k(J, b, t, h);
            const double bt = J->beta[row_s(J, b, t, h)];
            const double *dOt = J->dO ? J->dO + row_v(J, b, t, h) : NULL;
            const double *dut = J->du ? J->du + row_v(J, b, t, h) : NULL;

            /* o_t = S_t^T q_t */
            if (dOt) {
                for (int c = 0; c < DK; ++c)
                    for (int j = 0; j < DV; ++j) G[c * DV + j] += qt[c] * dOt[j];
            }
            if (J->dq) {
                double *dqt = J->dq + row_k(J, b, t, h);
                for (int c = 0; c < DK; ++c) {
                    double acc = 0.0;
                    if (dOt)
                        for (int j = 0; j < DV; ++j) acc += St[c * DV + j] * dOt[j];
                    dqt[c] = acc;
                }
            }
            /* S_t = S' + k u^T  and  u = beta (v - S'^T k) */
            for (int j = 0; j < DV; ++j) {
                double acc = dut ? dut[j] : 0.0;
                for (int c = 0; c < DK; ++c) acc += G[c * DV + j] * kt[c];
                dU[j] = acc;
            }
            if (J->dv) {
                double *dvt = J->dv + row_v(J, b, t, h);
                for (int j = 0; j < DV; ++j) dvt[j] = bt * dU[j];
            }
            if (J->dbeta) {
                double acc = 0.0;
                for (int j = 0; j < DV; ++j) acc += et[j] * dU[j];
                J->dbeta[row_s(J, b, t, h)] = acc;
            }
            if (J->dk) {
                double *dkt = J->dk + row_k(J, b, t, h);
                for (int c = 0; c < DK; ++c) {
                    double acc = 0.0;
                    for (int j = 0; j < DV; ++j) acc += G[c * DV + j] * ut[j] - bt * Sp[c * DV + j] * dU[j];
                    dkt[c] = acc;
                }
            }
            for (int c = 0; c < DK; ++c)
                for (int j = 0; j < DV; ++j) dSp[c * DV + j] = G[c * DV + j] - bt * kt[c] * dU[j];
            /* S' = Diag(alpha) S_{t-1} */
            if (J->dloga && J->variant != ORACLE_DELTANET) {
                if (J->variant == ORACLE_KDA) {
                    double *dl = J->dloga + row_k(J, b, t, h);
                    for (int c = 0; c < DK; ++c) {
                        double acc = 0.0;
                        for (int j = 0; j < DV; ++j) acc += dSp[c * DV + j] * Sp[c * DV + j];
                        dl[c] = acc;
                    }
                } else {
                    double acc = 0.0;
                    for (size_t x = 0; x < ns; ++x) acc += dSp[x] * Sp[x];
                    J->dloga[row_s(J, b, t, h)] = acc;
                }
            }
            for (int c = 0; c < DK; ++c) {
                const double a = gate(J, b, t, h, c);
                for (int j = 0; j < DV; ++j) G[c * DV + j] = a * dSp[c * DV + j];
            }
        }
    }
    if (J->dS0) memcpy(J->dS0 + state_off(J, b, h), G, sizeof(double) * ns);
done:
    free(ckpt); free(Sseg); free(Spseg); free(eseg); free(useg);
    free(S); free(G); free(dSp); free(dU);
    return rc;
}

/* ------------------------------------------------------------------------- */
/* chunkwise form, brute force                                                */
/* ------------------------------------------------------------------------- */
/*
 * Solve the dense n x n system M X = R (R has m columns, row-major) in place by
 * Gaussian elimination with partial pivoting.  M is destroyed; X overwrites R.
 */
static int dense_solve(double *M, double *R, int n, int m) {
    for (int p = 0; p < n; ++p) {
        int piv = p;
        for (int r = p + 1; r < n; ++r)
            if (fabs(M[r * n + p]) > fabs(M[piv * n + p])) piv = r;
        if (M[piv * n + p] == 0.0) return -1;
        if (piv != p) {
            for (int c = 0; c < n; ++c) { double t = M[p * n + c]; M[p * n + c] = M[piv * n + c]; M[piv * n + c] = t; }
            for (int c = 0; c < m; ++c) { double t = R[p * m + c]; R[p * m + c] = R[piv * m + c]; R[piv * m + c] = t; }
        }
        for (int r = p + 1; r < n; ++r) {
            const double f = M[r * n + p] / M[p * n + p];
            if (f == 0.0) continue;
            for (int c = p; c < n; ++c) M[r * n + c] -= f * M[p * n + c];
            for (int c = 0; c < m; ++c) R[r * m + c] -= f * R[p * m + c];
        }
    }
    for (int p = n - 1; p >= 0; --p) {
        for (int c = 0; c < m; ++c) {
            double acc = R[p * m + c];
            for (int r = p + 1; r < n; ++r) acc -= M[p * n + r] * R[r * m + c];
            R[p * m + c] = acc / M[p * n + p];
        }
    }
    return 0;
}

/*
 * One chunk of L tokens starting at t0, state S (dk x dv) updated in place.
 * g_r = sum_{i<=r} log alpha_i (per channel), gamma_r = exp(g_r).  Unrolling the
 * recurrence inside the chunk gives, for the write values u_r,
 *     u_r + beta_r sum_{i<r} (sum_c k_rc k_ic e^{g_rc - g_ic}) u_i
 *         = beta_r (v_r - (gamma_r .* k_r)^T S),
 * i.e. (I + A) U = diag(beta) (V - Ktil S) with A strictly lower triangular;
 * then
 *     o_r  = (gamma_r .* q_r)^T S + sum_{i<=r} (sum_c q_rc k_ic e^{g_rc - g_ic}) u_i,
 *     S   <- Diag(gamma_L) S + sum_r (k_r .* e^{g_L - g_r}) u_r^T.
 */
static int chunk_unit(job_t *J, int b, int h) {
    const int DK = J->DK, DV = J->DV, T = J->T, C = J->chunk;
    const size_t ns = (size_t)DK * DV;
    int rc = 0;
    double *S = malloc(sizeof(double) * ns);
    double *g = malloc(sizeof(double) * (size_t)C * DK);
    double *M = malloc(sizeof(double) * (size_t)C * C);
    double *R = malloc(sizeof(double) * (size_t)C * DV);
    double *Snew = malloc(sizeof(double) * ns);
    if (!S || !g || !M || !R || !Snew) { rc = -2; goto done; }
    load_initial_state(J, b, h, S);
    for (int t0 = 0; t0 < T; t0 += C) {
        const int L = (t0 + C <= T) ? C : T - t0;
        /* in-chunk cumulative log-gates */
        for (int r = 0; r < L; ++r)
            for (int c = 0; c < DK; ++c)
                g[r * DK + c] = (r ? g[(r - 1) * DK + c] : 0.0) + log_gate(J, b, t0 + r, h, c);
        /* system matrix I + A and right-hand side diag(beta)(V - Ktil S) */
        for (int r = 0; r < L; ++r) {
            const double *kr = J->k + row_k(J, b, t0 + r, h);
            const double br = J->beta[row_s(J, b, t0 + r, h)];
            for (int i = 0; i < L; ++i) {
                double a = 0.0;
                if (i < r) {
                    const double *ki = J->k + row_k(J, b, t0 + i, h);
                    for (int c = 0; c < DK; ++c) a += kr[c] * ki[c] * exp(g[r * DK + c] - g[i * DK + c]);
                    a *= br;
                }
                M[r * L + i] = (i == r ? 1.0 : 0.0) + a;
            }
            const double *vr = J->v + row_v(J, b, t0 + r, h);
            for (int j = 0; j < DV; ++j) {
                double ks = 0.0;
                for (int c = 0; c < DK; ++c) ks += exp(g[r * DK + c]) * kr[c] * S[c * DV + j];
                R[r * DV + j] = br * (vr[j] - ks);
            }
        }
        if (dense_solve(M, R, L, DV)) { rc = -1; goto done; }
        /* R now holds U (the write values of the chunk) */
        for (int r = 0; r < L; ++r) {
            if (J->u) memcpy(J->u + row_v(J, b, t0 + r, h), R + (size_t)r * DV, sizeof(double) * DV);
            if (J->o) {
                const double *qr = J->q + row_k(J, b, t0 + r, h);
                double *orow = J->o + row_v(J, b, t0 + r, h);
                for (int j = 0; j < DV; ++j) {
                    double acc = 0.0;
                    for (int c = 0; c < DK; ++c) acc += exp(g[r * DK + c]) * qr[c] * S[c * DV + j];
                    orow[j] = acc;
                }
                for (int i = 0; i <= r; ++i) {
                    const double *ki = J->k + row_k(J, b, t0 + i, h);
                    double p = 0.0;
                    for (int c = 0; c < DK; ++c) p += qr[c] * ki[c] * exp(g[r * DK + c] - g[i * DK + c]);
                    for (int j = 0; j < DV; ++j) orow[j] += p * R[i * DV + j];
                }
            }
        }
        /* state hand-off to the next chunk */
        for (int c = 0; c < DK; ++c) {
            const double gl = g[(L - 1) * DK + c];
            for (int j = 0; j < DV; ++j) {
                double acc = exp(gl) * S[c * DV + j];
                for (int r = 0; r < L; ++r) {
                    const double *kr = J->k + row_k(J, b, t0 + r, h);
                    acc += kr[c] * exp(gl - g[r * DK + c]) * R[r * DV + j];
                }
                Snew[c * DV + j] = acc;
            }
        }
        memcpy(S, Snew, sizeof(double) * ns);
    }
    if (J->ST) memcpy(J->ST + state_off(J, b, h), S, sizeof(double) * ns);
done:
    free(S); free(g); free(M); free(R); free(Snew);
    return rc;
}

/* ------------------------------------------------------------------------- */
/* threading over (b, h)                                                      */
/* ------------------------------------------------------------------------- */
typedef int (*unit_fn)(job_t *, int, int);
typedef struct { job_t *J; unit_fn fn; } worker_arg;

static void *worker(void *p) {
    worker_arg *w = (worker_arg *)p;
    job_t *J = w->J;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int unit = J->next_unit++;
        const int stop = J->failed;
        pthread_mutex_unlock(&J->lock);
        if (stop || unit >= J->B * J->H) break;
        const int rc = w->fn(J, unit / J->H, unit % J->H);
        if (rc) {
            pthread_mutex_lock(&J->lock);
            if (!J->failed) J->failed = rc;
            pthread_mutex_unlock(&J->lock);
        }
    }
    return NULL;
}

static int run(job_t *J, unit_fn fn, int nthreads) {
    if (J->B < 0 || J->T < 0 || J->H < 0 || J->DK < 1 || J->DV < 1) return -1;
    if (J->variant < ORACLE_DELTANET || J->variant > ORACLE_KDA) return -1;
    if (J->variant != ORACLE_DELTANET && !J->loga && J->T > 0 && J->B > 0 && J->H > 0) return -1;
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > J->B * J->H) nthreads = J->B * J->H > 0 ? J->B * J->H : 1;
    pthread_mutex_init(&J->lock, NULL);
    J->next_unit = 0;
    J->failed = 0;
    worker_arg w = {J, fn};
    pthread_t *th = malloc(sizeof(pthread_t) * nthreads);
    if (!th) return -2;
    int started = 0;
    for (int i = 0; i < nthreads; ++i)
        if (pthread_create(&th[i], NULL, worker, &w) == 0) ++started;
    if (started == 0) worker(&w);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J->lock);
    return J->failed;
}

int oracle_fwd(const double *q, const double *k, const double *v, const double *loga, const double *beta,
               const double *S0, double *o, double *u, double *ST, int B, int T, int H, int dk, int dv,
               int variant, int nthreads) {
    job_t J;
    memset(&J, 0, sizeof J);
    J.q = q; J.k = k; J.v = v; J.loga = loga; J.beta = beta; J.S0 = S0;
    J.o = o; J.u = u; J.ST = ST;
    J.B = B; J.T = T; J.H = H; J.DK = dk; J.DV = dv; J.variant = variant;
    return run(&J, fwd_unit, nthreads);
}

int oracle_bwd(const double *q, const double *k, const double *v, const double *loga, const double *beta,
               const double *S0, const double *dO, const double *du, const double *dST, double *dq, double *dk_,
               double *dv_, double *dloga, double *dbeta, double *dS0, int B, int T, int H, int dk, int dv,
               int variant, int nthreads) {
    job_t J;
    memset(&J, 0, sizeof J);
    J.q = q; J.k = k; J.v = v; J.loga = loga; J.beta = beta; J.S0 = S0;
    J.dO = dO; J.du = du; J.dST = dST;
    J.dq = dq; J.dk = dk_; J.dv = dv_; J.dloga = dloga; J.dbeta = dbeta; J.dS0 = dS0;
    J.B = B; J.T = T; J.H = H; J.DK = dk; J.DV = dv; J.variant = variant;
    return run(&J, bwd_unit, nthreads);
}

int oracle_chunked_fwd(const double *q, const double *k, const double *v, const double *loga, const double *beta,
                       const double *S0, double *o, double *u, double *ST, int B, int T, int H, int dk, int dv,
                       int variant, int chunk, int nthreads) {
    if (chunk < 1) return -1;
    job_t J;
    memset(&J, 0, sizeof J);
    J.q = q; J.k = k; J.v = v; J.loga = loga; J.beta = beta; J.S0 = S0;
    J.o = o; J.u = u; J.ST = ST;
    J.B = B; J.T = T; J.H = H; J.DK = dk; J.DV = dv; J.variant = variant; J.chunk = chunk;
    return run(&J, chunk_unit, nthreads);
}
