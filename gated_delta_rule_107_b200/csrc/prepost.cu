// prepost.cu -- the operations just before and just after the delta-rule core, each one
// pass over HBM ("线性注意力架构演进与Kimi Delta Attention创新实践": section 7.1 for the
// L2-normalised q, k and the logistic forget gate kept in log space, section 4.1 for the
// sigmoid output gate on RMSNorm of the core's output).
//
// Per (token, head) row, eps = 1e-6:
//   pre:   q_hat = q / sqrt(|q|^2 + eps),  k_hat likewise,  beta = sigmoid(b),
//          log alpha = -softplus(a)  (one a per row for Gated DeltaNet, one per key channel
//          for KDA, none for DeltaNet)
//   post:  y = o / sqrt(mean(o^2) + eps) * w * sigmoid(g)
// and their backward passes.  Every lane moves 16 bytes of a row, so a warp covers one to
// four rows at once (dk, dv in {64, 128}, fp32 or bf16); the post backward also sums w's gradient over all rows, deterministically: a fixed
// grid writes one partial per CTA, and a second kernel adds the partials in order.
#include "prepost.cuh"

namespace dr {
namespace pp {

constexpr float EPS = 1e-6f;
constexpr int WARPS = 8;            // rows in flight per CTA
constexpr int DW_CTAS = 1184;       // CTAs of the post backward (partials of dw): 8 per SM

// 16 bytes of consecutive elements (aligned to 16) in one access
template <typename E, int PL> struct Vec;
template <> struct Vec<float, 4> {
    static __device__ __forceinline__ void ld(const float *p, float *v) {
        const float4 x = *reinterpret_cast<const float4 *>(p);
        v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
    }
    static __device__ __forceinline__ void st(float *p, const float *v) {
        *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    }
};
template <> struct Vec<__nv_bfloat16, 8> {
    static __device__ __forceinline__ void ld(const __nv_bfloat16 *p, float *v) {
        const uint4 x = *reinterpret_cast<const uint4 *>(p);
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
    static __device__ __forceinline__ void st(__nv_bfloat16 *p, const float *v) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 a = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t *>(&a);
        }
        *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    }
};

// Row layout of a warp: each lane moves 16 bytes (VEC elements); LPR = D / VEC lanes share a
// row and a warp covers RPW = 32 / LPR rows at once.  sum_row() adds over a row's lanes.
template <typename E, int D> struct Lay {
    static constexpr int VEC = 16 / (int)sizeof(E), LPR = D / VEC, RPW = 32 / LPR;
};
template <int LPR> __device__ __forceinline__ float sum_row(float x) {
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ float sigmoid_f(float x) { return 1.f / (1.f + __expf(-x)); }
// softplus(x) = max(x, 0) + log(1 + e^{-|x|}), finite for every x
__device__ __forceinline__ float softplus_f(float x) { return fmaxf(x, 0.f) + log1pf(__expf(-fabsf(x))); }

// ------------------------------------------------------------------ pre
template <typename E, int VAR, int DK>
__global__ void __launch_bounds__(WARPS * 32) k_preop(const E *__restrict__ q, const E *__restrict__ k,
                                                      const E *__restrict__ b, const E *__restrict__ a,
                                                      E *__restrict__ qo, E *__restrict__ ko, E *__restrict__ bo,
                                                      E *__restrict__ ao, size_t rows) {
    using L = Lay<E, DK>;
    constexpr int PL = L::VEC;
    const int lane = threadIdx.x & 31, lr = lane % L::LPR;
    const size_t step = (size_t)gridDim.x * WARPS * L::RPW;
    for (size_t r0 = ((size_t)blockIdx.x * WARPS + (threadIdx.x >> 5)) * L::RPW; r0 < rows; r0 += step) {
        const size_t row = r0 + lane / L::LPR;
        const bool act = row < rows;
        const size_t base = row * DK + lr * PL;
        float xq[PL] = {}, xk[PL] = {}, sq = 0.f, sk = 0.f;
        if (act) {
            Vec<E, PL>::ld(q + base, xq);
            Vec<E, PL>::ld(k + base, xk);
        }
#pragma unroll
        for (int i = 0; i < PL; ++i) {
            sq += xq[i] * xq[i];
            sk += xk[i] * xk[i];
        }
        const float rq = rsqrtf(sum_row<L::LPR>(sq) + EPS), rk = rsqrtf(sum_row<L::LPR>(sk) + EPS);
        if (!act) continue;
#pragma unroll
        for (int i = 0; i < PL; ++i) {
            xq[i] *= rq;
            xk[i] *= rk;
        }
        Vec<E, PL>::st(qo + base, xq);
        Vec<E, PL>::st(ko + base, xk);
        if (VAR == VAR_KDA) {
            float xa[PL];
            Vec<E, PL>::ld(a + base, xa);
#pragma unroll
            for (int i = 0; i < PL; ++i) xa[i] = -softplus_f(xa[i]);
            Vec<E, PL>::st(ao + base, xa);
        }
        if (lr == 0) {
            bo[row] = from_f<E>(sigmoid_f(to_f(b[row])));
            if (VAR == VAR_GATED) ao[row] = from_f<E>(-softplus_f(to_f(a[row])));
        }
    }
}

template <typename E, int VAR, int DK>
__global__ void __launch_bounds__(WARPS * 32) k_preop_bwd(const E *__restrict__ q, const E *__restrict__ k,
                                                          const E *__restrict__ b, const E *__restrict__ a,
                                                          const E *__restrict__ dq, const E *__restrict__ dk,
                                                          const E *__restrict__ dbt, const E *__restrict__ dla,
                                                          E *__restrict__ gq, E *__restrict__ gk, E *__restrict__ gb,
                                                          E *__restrict__ ga, size_t rows) {
    using L = Lay<E, DK>;
    constexpr int PL = L::VEC;
    const int lane = threadIdx.x & 31, lr = lane % L::LPR;
    const size_t step = (size_t)gridDim.x * WARPS * L::RPW;
    for (size_t r0 = ((size_t)blockIdx.x * WARPS + (threadIdx.x >> 5)) * L::RPW; r0 < rows; r0 += step) {
        const size_t row = r0 + lane / L::LPR;
        const bool act = row < rows;
        const size_t base = row * DK + lr * PL;
        // d x = (dy - y (y . dy)) / r with y = x / r, r = sqrt(|x|^2 + eps), for x = q and x = k
        float xq[PL] = {}, xk[PL] = {}, yq[PL] = {}, yk[PL] = {}, sq = 0.f, sk = 0.f, pq = 0.f, pk = 0.f;
        if (act) {
            Vec<E, PL>::ld(q + base, xq);
            Vec<E, PL>::ld(k + base, xk);
            Vec<E, PL>::ld(dq + base, yq);
            Vec<E, PL>::ld(dk + base, yk);
        }
#pragma unroll
        for (int i = 0; i < PL; ++i) {
            sq += xq[i] * xq[i];
            sk += xk[i] * xk[i];
            pq += xq[i] * yq[i];
            pk += xk[i] * yk[i];
        }
        const float rq = rsqrtf(sum_row<L::LPR>(sq) + EPS), rk = rsqrtf(sum_row<L::LPR>(sk) + EPS);
        const float cq = sum_row<L::LPR>(pq) * rq * rq, ck = sum_row<L::LPR>(pk) * rk * rk;  // (y . dy) / r
        if (!act) continue;
#pragma unroll
        for (int i = 0; i < PL; ++i) {
            yq[i] = (yq[i] - xq[i] * cq) * rq;
            yk[i] = (yk[i] - xk[i] * ck) * rk;
        }
        Vec<E, PL>::st(gq + base, yq);
        Vec<E, PL>::st(gk + base, yk);
        if (VAR == VAR_KDA) {
            float xa[PL], ya[PL];
            Vec<E, PL>::ld(a + base, xa);
            Vec<E, PL>::ld(dla + base, ya);
#pragma unroll
            for (int i = 0; i < PL; ++i) ya[i] = -ya[i] * sigmoid_f(xa[i]);
            Vec<E, PL>::st(ga + base, ya);
        }
        if (lr == 0) {
            const float s = sigmoid_f(to_f(b[row]));
            gb[row] = from_f<E>(to_f(dbt[row]) * s * (1.f - s));
            if (VAR == VAR_GATED) ga[row] = from_f<E>(-to_f(dla[row]) * sigmoid_f(to_f(a[row])));
        }
    }
}

// ------------------------------------------------------------------ post
template <typename E, int DV>
__global__ void __launch_bounds__(WARPS * 32) k_postop(const E *__restrict__ o, const E *__restrict__ g,
                                                       const float *__restrict__ w, E *__restrict__ y, size_t rows) {
    using L = Lay<E, DV>;
    constexpr int PL = L::VEC;
    const int lane = threadIdx.x & 31, lr = lane % L::LPR;
    float wl[PL];
#pragma unroll
    for (int i = 0; i < PL; ++i) wl[i] = w ? w[lr * PL + i] : 1.f;
    const size_t step = (size_t)gridDim.x * WARPS * L::RPW;
    for (size_t r0 = ((size_t)blockIdx.x * WARPS + (threadIdx.x >> 5)) * L::RPW; r0 < rows; r0 += step) {
        const size_t row = r0 + lane / L::LPR;
        const bool act = row < rows;
        const size_t base = row * DV + lr * PL;
        float x[PL] = {}, gx[PL] = {}, ss = 0.f;
        if (act) {
            Vec<E, PL>::ld(o + base, x);
            Vec<E, PL>::ld(g + base, gx);
        }
#pragma unroll
        for (int i = 0; i < PL; ++i) ss += x[i] * x[i];
        const float r = rsqrtf(sum_row<L::LPR>(ss) * (1.f / DV) + EPS);
        if (!act) continue;
#pragma unroll
        for (int i = 0; i < PL; ++i) x[i] *= r * wl[i] * sigmoid_f(gx[i]);
        Vec<E, PL>::st(y + base, x);
    }
}

// dw partial of this CTA -> part[blockIdx.x][DV]
template <typename E, int DV>
__global__ void __launch_bounds__(WARPS * 32) k_postop_bwd(const E *__restrict__ o, const E *__restrict__ g,
                                                           const float *__restrict__ w, const E *__restrict__ dy,
                                                           E *__restrict__ go, E *__restrict__ gg,
                                                           float *__restrict__ part, size_t rows) {
    using L = Lay<E, DV>;
    constexpr int PL = L::VEC;
    __shared__ float acc[WARPS][DV];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, lr = lane % L::LPR;
    float wl[PL], dwl[PL];
#pragma unroll
    for (int i = 0; i < PL; ++i) {
        wl[i] = w ? w[lr * PL + i] : 1.f;
        dwl[i] = 0.f;
    }
    const size_t step = (size_t)gridDim.x * WARPS * L::RPW;
    for (size_t r0 = ((size_t)blockIdx.x * WARPS + warp) * L::RPW; r0 < rows; r0 += step) {
        const size_t row = r0 + lane / L::LPR;
        const bool act = row < rows;
        const size_t base = row * DV + lr * PL;
        float x[PL] = {}, gy[PL] = {}, s[PL] = {}, ss = 0.f;
        if (act) {
            Vec<E, PL>::ld(o + base, x);
            Vec<E, PL>::ld(dy + base, gy);
            Vec<E, PL>::ld(g + base, s);
        }
#pragma unroll
        for (int i = 0; i < PL; ++i) {
            s[i] = sigmoid_f(s[i]);
            ss += x[i] * x[i];
        }
        const float r = rsqrtf(sum_row<L::LPR>(ss) * (1.f / DV) + EPS);
        // n = x r;  dz = dy s;  dg = dy n w s (1 - s);  dw += dz n;  dn = dz w;
        // do = r (dn - n mean(dn n))   (inactive rows carry zeros throughout)
        float dn[PL], dgv[PL], pn = 0.f;
#pragma unroll
        for (int i = 0; i < PL; ++i) {
            const float n = x[i] * r, dz = gy[i] * s[i];
            dgv[i] = dz * n * wl[i] * (1.f - s[i]);
            dwl[i] += dz * n;
            dn[i] = dz * wl[i];
            pn += dn[i] * n;
        }
        const float m = sum_row<L::LPR>(pn) * (1.f / DV);
        if (!act) continue;
        Vec<E, PL>::st(gg + base, dgv);
#pragma unroll
        for (int i = 0; i < PL; ++i) dn[i] = r * (dn[i] - x[i] * r * m);
        Vec<E, PL>::st(go + base, dn);
    }
    // lanes that share columns (one per row of the warp) add up, then the warps in order
#pragma unroll
    for (int i = 0; i < PL; ++i) {
        for (int o2 = L::LPR; o2 < 32; o2 <<= 1) dwl[i] += __shfl_xor_sync(0xffffffffu, dwl[i], o2);
    }
    if (lane < L::LPR) {
#pragma unroll
        for (int i = 0; i < PL; ++i) acc[warp][lr * PL + i] = dwl[i];
    }
    __syncthreads();
    for (int c = threadIdx.x; c < DV; c += WARPS * 32) {
        float t = 0.f;
#pragma unroll
        for (int wp = 0; wp < WARPS; ++wp) t += acc[wp][c];
        part[(size_t)blockIdx.x * DV + c] = t;
    }
}

// dw[c] = sum over the partials: thread (c, s) adds partials s, s + 8, ... in order, then
// the eight sums are added in order (a fixed order: deterministic)
template <int DV>
__global__ void __launch_bounds__(DV * 8) k_postop_dw(const float *__restrict__ part, int nparts,
                                                      float *__restrict__ dw) {
    __shared__ float acc[8][DV];
    const int c = threadIdx.x % DV, sl = threadIdx.x / DV;
    float t = 0.f;
    for (int p = sl; p < nparts; p += 8) t += part[(size_t)p * DV + c];
    acc[sl][c] = t;
    __syncthreads();
    if (sl == 0) {
        float u = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) u += acc[i][c];
        dw[c] = u;
    }
}

// CTAs for rows spread rows_per_cta to a CTA (grid-stride loops cover any remainder)
inline unsigned grid_for(size_t rows, int rows_per_cta) {
    const size_t want = (rows + rows_per_cta - 1) / rows_per_cta;
    return (unsigned)(want < 65535u * 16u ? want : 65535u * 16u);
}

template <typename E, int VAR>
cudaError_t pre_v(const PrePost &p, bool bwd, cudaStream_t s) {
    const unsigned grid = grid_for(p.rows, WARPS * (p.d == 128 ? Lay<E, 128>::RPW : Lay<E, 64>::RPW));
    const E *q = (const E *)p.q, *k = (const E *)p.k, *b = (const E *)p.b, *a = (const E *)p.a;
    if (!bwd) {
        if (p.d == 128)
            k_preop<E, VAR, 128><<<grid, WARPS * 32, 0, s>>>(q, k, b, a, (E *)p.qo, (E *)p.ko, (E *)p.bo, (E *)p.ao,
                                                            p.rows);
        else
            k_preop<E, VAR, 64><<<grid, WARPS * 32, 0, s>>>(q, k, b, a, (E *)p.qo, (E *)p.ko, (E *)p.bo, (E *)p.ao,
                                                           p.rows);
    } else {
        const E *dq = (const E *)p.dq, *dk = (const E *)p.dk, *db = (const E *)p.db, *da = (const E *)p.da;
        if (p.d == 128)
            k_preop_bwd<E, VAR, 128><<<grid, WARPS * 32, 0, s>>>(q, k, b, a, dq, dk, db, da, (E *)p.qo, (E *)p.ko,
                                                                (E *)p.bo, (E *)p.ao, p.rows);
        else
            k_preop_bwd<E, VAR, 64><<<grid, WARPS * 32, 0, s>>>(q, k, b, a, dq, dk, db, da, (E *)p.qo, (E *)p.ko,
                                                               (E *)p.bo, (E *)p.ao, p.rows);
    }
    return cudaGetLastError();
}

template <typename E>
cudaError_t pre_e(const PrePost &p, bool bwd, cudaStream_t s) {
    if (p.variant == VAR_GATED) return pre_v<E, VAR_GATED>(p, bwd, s);
    if (p.variant == VAR_KDA) return pre_v<E, VAR_KDA>(p, bwd, s);
    return pre_v<E, VAR_DELTANET>(p, bwd, s);
}

template <typename E, int DV>
cudaError_t post_d(const PrePost &p, bool bwd, cudaStream_t s) {
    const E *o = (const E *)p.q, *g = (const E *)p.k;
    if (!bwd) {
        k_postop<E, DV><<<grid_for(p.rows, WARPS * Lay<E, DV>::RPW), WARPS * 32, 0, s>>>(o, g, p.w, (E *)p.qo, p.rows);
        return cudaGetLastError();
    }
    k_postop_bwd<E, DV><<<DW_CTAS, WARPS * 32, 0, s>>>(o, g, p.w, (const E *)p.dq, (E *)p.qo, (E *)p.ko, p.part,
                                                       p.rows);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || !p.dw) return e;
    k_postop_dw<DV><<<1, DV * 8, 0, s>>>(p.part, DW_CTAS, p.dw);
    return cudaGetLastError();
}

}  // namespace pp

size_t postop_ws_bytes(int dv) { return (size_t)pp::DW_CTAS * dv * sizeof(float); }

cudaError_t preop_run(const PrePost &p, bool bf16, bool bwd, cudaStream_t s) {
    return bf16 ? pp::pre_e<__nv_bfloat16>(p, bwd, s) : pp::pre_e<float>(p, bwd, s);
}

cudaError_t postop_run(const PrePost &p, bool bf16, bool bwd, cudaStream_t s) {
    if (p.d == 128) return bf16 ? pp::post_d<__nv_bfloat16, 128>(p, bwd, s) : pp::post_d<float, 128>(p, bwd, s);
    return bf16 ? pp::post_d<__nv_bfloat16, 64>(p, bwd, s) : pp::post_d<float, 64>(p, bwd, s);
}

}  // namespace dr
