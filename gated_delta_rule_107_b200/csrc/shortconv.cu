// shortconv.cu -- depthwise causal convolution of kernel size 4 over the token axis
// ("线性注意力架构演进与Kimi Delta Attention创新实践", section 4.2: a kernel-4 depthwise
// convolution on the q/k/v path), forward and backward, one pass over HBM each.
//
// For a token-major stream x [B, T, D] and per-channel taps w [D][4] (fp32, the last tap on the
// current token), with x at t < 0 read from the three-token cache x_prev [B, 3, D] or zero:
//   y[b, t, c]  = sum_j w[c][j] x[b, t - 3 + j, c]
//   dx[b, s, c] = sum_j w[c][j] dy[b, s + 3 - j, c]      (s = -3 .. T-1; s < 0 is dx_prev)
//   dw[c][j]    = sum_{b, t} dy[b, t, c] x[b, t - 3 + j, c]
// A thread owns a group of channels of one sequence (16 bytes in the forward, 4 channels in the
// backward) and walks a block of tokens with the three neighbouring rows in registers, so every
// element is read once, plus a three-row halo per block; a warp's lanes hold consecutive
// channel groups of one token, rows are loaded 8 at a time before any is used.  The backward sums dw per token block into a partial; a second
// kernel adds the partials in a fixed order, so dw is deterministic.
#include "shortconv.cuh"

namespace dr {
namespace scv {

constexpr int K = 4;      // taps
constexpr int NT = 256;   // threads per CTA
constexpr int TBF = 32;   // tokens per thread, forward
constexpr int TBB = 64;   // tokens per thread, backward (one dw partial per block)

inline int blocks_of(int T, int tb) { return T <= 0 ? 1 : (T + tb - 1) / tb; }

constexpr int BATF = 8;   // rows loaded together (packed vectors) before any is used, forward
constexpr int BATB = 8;   // the same for each of dy and x, backward

// VB bytes of consecutive elements (aligned to VB) of one row: the forward moves 16 bytes a
// lane, the backward 4 elements a lane (8 bytes of bf16), which halves its registers
template <typename E, int VB> struct Lane;
template <> struct Lane<float, 16> {
    static constexpr int PL = 4;
    using Raw = uint4;
    static __device__ __forceinline__ Raw zero() { return make_uint4(0u, 0u, 0u, 0u); }
    static __device__ __forceinline__ void unpack(const Raw &r, float *v) {
        v[0] = __uint_as_float(r.x); v[1] = __uint_as_float(r.y);
        v[2] = __uint_as_float(r.z); v[3] = __uint_as_float(r.w);
    }
    static __device__ __forceinline__ void st(float *p, const float *v) {
        *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    }
};
template <> struct Lane<__nv_bfloat16, 16> {
    static constexpr int PL = 8;
    using Raw = uint4;
    static __device__ __forceinline__ Raw zero() { return make_uint4(0u, 0u, 0u, 0u); }
    static __device__ __forceinline__ void unpack(const Raw &r, float *v) {
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
    static __device__ __forceinline__ void st(__nv_bfloat16 *p, const float *v) { pp::Vec<__nv_bfloat16, 8>::st(p, v); }
};
template <> struct Lane<__nv_bfloat16, 8> {
    static constexpr int PL = 4;
    using Raw = uint2;
    static __device__ __forceinline__ Raw zero() { return make_uint2(0u, 0u); }
    static __device__ __forceinline__ void unpack(const Raw &r, float *v) {
        v[0] = __uint_as_float(r.x << 16); v[1] = __uint_as_float(r.x & 0xFFFF0000u);
        v[2] = __uint_as_float(r.y << 16); v[3] = __uint_as_float(r.y & 0xFFFF0000u);
    }
    static __device__ __forceinline__ void st(__nv_bfloat16 *p, const float *v) {
        const __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]);
        *reinterpret_cast<uint2 *>(p) =
            make_uint2(*reinterpret_cast<const uint32_t *>(&a), *reinterpret_cast<const uint32_t *>(&b));
    }
};
template <typename E> constexpr int fwd_vb() { return 16; }
template <typename E> constexpr int bwd_vb() { return 4 * (int)sizeof(E); }

template <typename E, int VB>
__device__ __forceinline__ typename Lane<E, VB>::Raw ldv(const E *p) {
    return *reinterpret_cast<const typename Lane<E, VB>::Raw *>(p);
}

// token t of sequence b at channel offset c0, packed (t < 0: the cache row 3 + t, or zeros)
template <typename E, int VB>
__device__ __forceinline__ typename Lane<E, VB>::Raw x_raw(const E *x, const E *cin, int b, int t, int T, int D,
                                                          int c0) {
    if (t >= 0) return ldv<E, VB>(x + ((size_t)b * T + t) * D + c0);
    if (cin) return ldv<E, VB>(cin + ((size_t)b * (K - 1) + (K - 1 + t)) * D + c0);
    return Lane<E, VB>::zero();
}

template <typename E>
__global__ void __launch_bounds__(NT) k_shortconv(const E *__restrict__ x, const float *__restrict__ w,
                                                  const E *__restrict__ cin, E *__restrict__ y, E *__restrict__ cout,
                                                  int B, int T, int D, int NTB) {
    constexpr int VB = fwd_vb<E>();
    using R = Lane<E, VB>;
    constexpr int PL = R::PL;
    const int NV = D / PL;
    const long long gid = (long long)blockIdx.x * NT + threadIdx.x;
    if (gid >= (long long)B * NTB * NV) return;
    const int cv = (int)(gid % NV);
    const long long bt = gid / NV;
    const int tb = (int)(bt % NTB), b = (int)(bt / NTB), c0 = cv * PL;
    const int t0 = tb * TBF, t1 = min(T, t0 + TBF);
    float h3[PL], h2[PL], h1[PL];  // tokens t - 3, t - 2, t - 1
    R::unpack(x_raw<E, VB>(x, cin, b, t0 - 3, T, D, c0), h3);
    R::unpack(x_raw<E, VB>(x, cin, b, t0 - 2, T, D, c0), h2);
    R::unpack(x_raw<E, VB>(x, cin, b, t0 - 1, T, D, c0), h1);
    float wr[K][PL];
#pragma unroll
    for (int i = 0; i < PL; ++i)
#pragma unroll
        for (int j = 0; j < K; ++j) wr[j][i] = w[(size_t)(c0 + i) * K + j];
    for (int s0 = t0; s0 < t1; s0 += BATF) {
        typename R::Raw raw[BATF];
#pragma unroll
        for (int e = 0; e < BATF; ++e)
            raw[e] = s0 + e < t1 ? ldv<E, VB>(x + ((size_t)b * T + s0 + e) * D + c0) : R::zero();
#pragma unroll
        for (int e = 0; e < BATF; ++e) {
            float xc[PL], o[PL];
            R::unpack(raw[e], xc);
#pragma unroll
            for (int i = 0; i < PL; ++i) {
                o[i] = wr[0][i] * h3[i] + wr[1][i] * h2[i] + wr[2][i] * h1[i] + wr[3][i] * xc[i];
                h3[i] = h2[i];
                h2[i] = h1[i];
                h1[i] = xc[i];
            }
            if (s0 + e < t1) R::st(y + ((size_t)b * T + s0 + e) * D + c0, o);
        }
    }
    if (cout && tb == NTB - 1) {  // the last three tokens of [x_prev ; x]
#pragma unroll
        for (int j = 0; j < K - 1; ++j) {
            const typename R::Raw r = x_raw<E, VB>(x, cin, b, T - (K - 1) + j, T, D, c0);
            *reinterpret_cast<typename R::Raw *>(cout + ((size_t)b * (K - 1) + j) * D + c0) = r;
        }
    }
}

// walks its block from the last token down (and, in the first block, on through the three cache
// positions when dcin is wanted); part[(b NTB + tb) D + c][j] = this block's share of dw[c][j]
template <typename E>
__global__ void __launch_bounds__(NT) k_shortconv_bwd(const E *__restrict__ x, const float *__restrict__ w,
                                                      const E *__restrict__ cin, const E *__restrict__ dy,
                                                      E *__restrict__ dx, E *__restrict__ dcin,
                                                      float *__restrict__ part, int B, int T, int D, int NTB) {
    constexpr int VB = bwd_vb<E>();
    using R = Lane<E, VB>;
    constexpr int PL = R::PL;
    const int NV = D / PL;
    const long long gid = (long long)blockIdx.x * NT + threadIdx.x;
    if (gid >= (long long)B * NTB * NV) return;
    const int cv = (int)(gid % NV);
    const long long bt = gid / NV;
    const int tb = (int)(bt % NTB), b = (int)(bt / NTB), c0 = cv * PL;
    const int t0 = tb * TBB, t1 = min(T, t0 + TBB);
    auto dy_raw = [&](int t) { return t < T ? ldv<E, VB>(dy + ((size_t)b * T + t) * D + c0) : R::zero(); };
    float g1[PL], g2[PL], g3[PL];  // dy at t + 1, t + 2, t + 3
    R::unpack(dy_raw(t1), g1);
    R::unpack(dy_raw(t1 + 1), g2);
    R::unpack(dy_raw(t1 + 2), g3);
    float a0[PL], a1[PL], a2[PL];  // x at t, t - 1, t - 2
    R::unpack(x_raw<E, VB>(x, cin, b, t1 - 1, T, D, c0), a0);
    R::unpack(x_raw<E, VB>(x, cin, b, t1 - 2, T, D, c0), a1);
    R::unpack(x_raw<E, VB>(x, cin, b, t1 - 3, T, D, c0), a2);
    float wr[K][PL], dwl[K][PL];
#pragma unroll
    for (int i = 0; i < PL; ++i)
#pragma unroll
        for (int j = 0; j < K; ++j) {
            wr[j][i] = w[(size_t)(c0 + i) * K + j];
            dwl[j][i] = 0.f;
        }
    for (int s1 = t1; s1 > t0; s1 -= BATB) {  // tokens s1 - 1 down to s1 - BATB (not below t0)
        typename R::Raw rdy[BATB], rx[BATB];
#pragma unroll
        for (int e = 0; e < BATB; ++e) {
            const int t = s1 - 1 - e;
            rdy[e] = t >= t0 ? ldv<E, VB>(dy + ((size_t)b * T + t) * D + c0) : R::zero();
            rx[e] = t >= t0 ? x_raw<E, VB>(x, cin, b, t - 3, T, D, c0) : R::zero();
        }
#pragma unroll
        for (int e = 0; e < BATB; ++e) {
            const int t = s1 - 1 - e;
            if (t < t0) break;
            float gt[PL], a3[PL], o[PL];
            R::unpack(rdy[e], gt);
            R::unpack(rx[e], a3);
#pragma unroll
            for (int i = 0; i < PL; ++i) {
                o[i] = wr[3][i] * gt[i] + wr[2][i] * g1[i] + wr[1][i] * g2[i] + wr[0][i] * g3[i];
                dwl[3][i] += gt[i] * a0[i];
                dwl[2][i] += gt[i] * a1[i];
                dwl[1][i] += gt[i] * a2[i];
                dwl[0][i] += gt[i] * a3[i];
                a0[i] = a1[i];
                a1[i] = a2[i];
                a2[i] = a3[i];
                g3[i] = g2[i];
                g2[i] = g1[i];
                g1[i] = gt[i];
            }
            R::st(dx + ((size_t)b * T + t) * D + c0, o);
        }
    }
    if (dcin && tb == 0) {  // positions -1, -2, -3: dy is zero there, the window carries on
#pragma unroll
        for (int s = -1; s >= -(K - 1); --s) {
            float o[PL];
#pragma unroll
            for (int i = 0; i < PL; ++i) {
                o[i] = wr[2][i] * g1[i] + wr[1][i] * g2[i] + wr[0][i] * g3[i];
                g3[i] = g2[i];
                g2[i] = g1[i];
                g1[i] = 0.f;
            }
            R::st(dcin + ((size_t)b * (K - 1) + (K - 1 + s)) * D + c0, o);
        }
    }
    if (part) {
        float *pp_ = part + ((size_t)(b * NTB + tb) * D + c0) * K;
#pragma unroll
        for (int i = 0; i < PL; ++i)
#pragma unroll
            for (int j = 0; j < K; ++j) pp_[i * K + j] = dwl[j][i];
    }
}

// dw[e] (e over D K) = sum of the P partials: thread (e, s) adds partials s, s + 8, ... in order,
// then the eight slices are added in order
__global__ void __launch_bounds__(NT) k_shortconv_dw(const float *__restrict__ part, int P, int n,
                                                     float *__restrict__ dw) {
    __shared__ float acc[8][NT / 8];
    const int el = threadIdx.x % (NT / 8), sl = threadIdx.x / (NT / 8);
    const int e = blockIdx.x * (NT / 8) + el;
    float t = 0.f;
    if (e < n) {
#pragma unroll 8
        for (int p = sl; p < P; p += 8) t += part[(size_t)p * n + e];
    }
    acc[sl][el] = t;
    __syncthreads();
    if (sl == 0 && e < n) {
        float u = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) u += acc[i][el];
        dw[e] = u;
    }
}

template <typename E>
cudaError_t run(const ShortConv &p, bool bwd, cudaStream_t s) {
    const long long ctas = shortconv_ctas(p.B, p.T, p.D, sizeof(E) == 2, bwd);
    if (ctas == 0) return cudaSuccess;
    const int NTB = blocks_of(p.T, bwd ? TBB : TBF);
    if (!bwd) {
        k_shortconv<E><<<(unsigned)ctas, NT, 0, s>>>((const E *)p.x, p.w, (const E *)p.cin, (E *)p.y, (E *)p.cout,
                                                     p.B, p.T, p.D, NTB);
        return cudaGetLastError();
    }
    float *part = p.dw ? p.part : nullptr;
    k_shortconv_bwd<E><<<(unsigned)ctas, NT, 0, s>>>((const E *)p.x, p.w, (const E *)p.cin, (const E *)p.dy,
                                                     (E *)p.dx, (E *)p.dcin, part, p.B, p.T, p.D, NTB);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || !p.dw) return e;
    const int n = p.D * K;
    k_shortconv_dw<<<(n + NT / 8 - 1) / (NT / 8), NT, 0, s>>>(p.part, p.B * NTB, n, p.dw);
    return cudaGetLastError();
}

}  // namespace scv

size_t shortconv_ws_bytes(int B, int T, int D) {
    return (size_t)B * scv::blocks_of(T, scv::TBB) * D * scv::K * sizeof(float);
}

long long shortconv_ctas(int B, int T, int D, bool bf16, bool bwd) {
    if (B <= 0 || D <= 0) return 0;
    const int per_lane = bwd ? 4 : (bf16 ? 8 : 4);  // channels a thread owns
    const long long threads = (long long)B * scv::blocks_of(T, bwd ? scv::TBB : scv::TBF) * (D / per_lane);
    return (threads + scv::NT - 1) / scv::NT;
}

cudaError_t shortconv_run(const ShortConv &p, bool bf16, bool bwd, cudaStream_t s) {
    return bf16 ? scv::run<__nv_bfloat16>(p, bwd, s) : scv::run<float>(p, bwd, s);
}

}  // namespace dr
