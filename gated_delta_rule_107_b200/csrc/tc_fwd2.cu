// tc_fwd2.cu -- warp-specialised fused forward for Gated DeltaNet and DeltaNet (sm_100a).
//
// Same per-chunk algebra as tc_fwd.cu ("线性注意力架构演进与Kimi Delta Attention创新实践",
// sections 2.1, 6.1, 6.2, 7.1), reorganised so that the preparation of chunk m+1 runs
// while the state chain processes chunk m:
//
//   warp 0       producer: TMA loads of k and q (interleaved per 64-channel panel so
//                that [k ; q] is one 128-row operand), of v, and plain loads of the
//                scalar gate and beta
//   warps 1-4    preparation warpgroup, per chunk:
//                  P1  [k ; q] . k^T                -> k.k^T, q.k^T   (TMEM)
//                      A = beta_r e^{g_r-g_i} k_r.k_i (i<r), P = e^{g_r-g_i} q_r.k_i (i<=r)
//                  T = (I + A)^-1                    (tc_inverse.cuh)
//                  IPT [I ; P] . T = R = [T ; P T]
//                  P3  (R diag(beta e^g)) . k       = [W ; P W]
//                  P4  (R diag(beta))     . v       = [U~ ; P U~]  -> accumulator D[m%2]
//                  A_chain = [-W ; e^g q - P W]
//   warps 5-8    chain warpgroup, per chunk:
//                  C1  D += A_chain . S             -> rows 0-63 U, rows 64-127 O
//                  C3  E = k^T . (e^{g_C - g} U)    (the decay to the chunk end is
//                                                     applied to U's rows, not to k)
//                  S <- e^{g_C} S + E               (fp32 registers)
//
// The gate enters only as row / column multipliers in epilogues: e^{g_r - g_i} is
// split at the chunk midpoint g_m into e^{g_r - g_m} e^{g_m - g_i}; a chunk whose
// cumulative log gate strays more than 80 from g_m uses exact per-pair exponentials.
// Hand-offs between the warpgroups are mbarriers; the accumulator D is double-buffered
// in TMEM; every wait is bounded (~1 s) and aborts are agreed on per warpgroup.
#include "tc_host.cuh"
#include "tc_inverse.cuh"
#include "tc_path.cuh"
#include "tc_ptx.cuh"
#include "tc_tile.cuh"
#include "simt_path.cuh"

namespace dr {
namespace tcf2 {

using namespace dr::tc;
using dr::tcf::ld_chunk;
using dr::tcf::st_chunk;
using dr::tcf::tmem_row64;

constexpr int C = 64, DK = 128, DVB = 64;
constexpr int NTHREADS = 288;

// ---- shared memory (bytes from a 1024-aligned base) ----
constexpr uint32_t SLOT = 32768;                 // [k_p0 | q_p0 | k_p1 | q_p1], 8K each
constexpr uint32_t OFF_V = 2 * SLOT;             //  8K  v (64 tokens x 64)
constexpr uint32_t OFF_KC = OFF_V + 8192;        // 2 x 16K  chain copy of k (2 panels of 8K)
constexpr uint32_t OFF_RR = OFF_KC + 32768;      // 32K  R diag(beta) | R diag(beta e^g); inverse scratch
constexpr uint32_t OFF_IP = OFF_RR + 32768;      // 16K  [I ; P]
constexpr uint32_t OFF_TT = OFF_IP + 16384;      //  8K  T (MN-major B)
constexpr uint32_t OFF_AC = OFF_TT + 8192;       // 32K  A_chain (128 rows x 2 panels of 16K)
constexpr uint32_t OFF_U = OFF_AC + 32768;       //  8K  e^{g_C - g} U
constexpr uint32_t OFF_S = OFF_U + 8192;         // 16K  bf16 S
constexpr uint32_t OFF_MISC = OFF_S + 16384;     //  8K
constexpr uint32_t SMEM_BYTES = OFF_MISC + 8192;

// misc
constexpr uint32_t M_BAR = 0;        // 16 mbarriers
constexpr uint32_t M_TMEM = 128, M_ABORT = 132, M_BIG = 136;  // M_BIG: int[2], per slot
constexpr uint32_t M_PF = 256;       // prep factors [2 slots][7][64]
constexpr uint32_t M_CF = 3840;      // chain factors [2][80]: e^{gC-g} (64), e^{gC}
constexpr uint32_t M_YS = 4608;      // inverse scratch [3][256]
static_assert(M_YS + 3 * 256 * 4 <= 8192, "misc overflow");
enum { PF_GC = 0, PF_ROWA, PF_ROWP, PF_COLA, PF_BV, PF_BK, PF_EG };

// TMEM columns
constexpr uint32_t TM_G1 = 0, TM_X = 64, TM_D0 = 192, TM_E = 320, TM_G = 384, TM_COLS = 512;

enum {
    B_FULL0 = 0, B_FULL1, B_EMPTY0, B_EMPTY1, B_VFULL, B_VEMPTY, B_PMMA, B_CMMA,
    B_READY0, B_READY1, B_ACFREE, B_DFREE0, B_DFREE1, B_KCFREE0, B_KCFREE1, B_NUM
};

struct Args {
    const void *alpha, *beta;
    const float *S0;
    void *out, *u;
    float *ST;
    int B, T, H, dv, N;
    // recompute mode (backward): the chunk products of the tensor-core backward workspace
    __nv_bfloat16 *W, *Ut, *P, *Sn, *Un, *Tn, *KK;
    float *G;
    // reverse mode: dL/dS of the state leaving each chunk; whether du is given
    __nv_bfloat16 *dSn;
    int has_du;
};

// 8 values as bf16 at element offset elem_off (a multiple of 8) of a bf16 array
__device__ __forceinline__ void st8_global(void *base, size_t elem_off, const float *v) {
    uint4 w;
    w.x = pack_bf16(v[0], v[1]);
    w.y = pack_bf16(v[2], v[3]);
    w.z = pack_bf16(v[4], v[5]);
    w.w = pack_bf16(v[6], v[7]);
    *reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(base) + elem_off) = w;
}

// 64 values as bf16 at element offset elem_off (a multiple of 8) of a bf16 array
__device__ __forceinline__ void st_row_global(void *base, size_t elem_off, const float *v) {
    uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(base) + elem_off);
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
        uint4 w;
        w.x = pack_bf16(v[ch * 8 + 0], v[ch * 8 + 1]);
        w.y = pack_bf16(v[ch * 8 + 2], v[ch * 8 + 3]);
        w.z = pack_bf16(v[ch * 8 + 4], v[ch * 8 + 5]);
        w.w = pack_bf16(v[ch * 8 + 6], v[ch * 8 + 7]);
        dst[ch] = w;
    }
}

// MODE 0: forward (o, u, S_T).
// MODE 1: recompute for the backward -- no o / u / S_T; instead g, k k^T, P, T, W, U~,
//         the entering state S_n and the write values U are stored (bf16 rows, fp32 g)
//         in the chunk-major layout of TcBwdWs.
// MODE 2: the backward's reverse state chain.  Chunks are visited last to first; the
//         preparation is the same (A_chain = [-W ; Q~ - P W]) minus P4, the chain's copy
//         of k is scaled to Kbar = e^{g_C - g} k, and the chain warpgroup evaluates
//           dS_n = e^{g_C} dS_{n+1} + A_chain^T [du ; dO] + ((-W)^T Kbar) dS_{n+1}
//         (= e^{g_C} dS+ + Qtil^T dO - W^T dU with dU = du + P^T dO + Kbar dS+),
//         storing dS_{n+1} for every chunk and dS_0 at the end.  S0 / S_T carry dS_T / dS0,
//         the v map carries dO and the x map du.
template <int VAR, int MODE>
__global__ void __launch_bounds__(NTHREADS, 1)
    k_fwd_tc2(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_x, Args a) {
    constexpr int SAVE = (MODE == 1);
    constexpr bool REV = (MODE == 2);
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + OFF_MISC + M_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC + M_TMEM);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + OFF_MISC + M_ABORT);
    volatile int *bigflag = reinterpret_cast<volatile int *>(sm + OFF_MISC + M_BIG);
    float *pf_all = reinterpret_cast<float *>(sm + OFF_MISC + M_PF);
    float *cf = reinterpret_cast<float *>(sm + OFF_MISC + M_CF);
    float *ysc = reinterpret_cast<float *>(sm + OFF_MISC + M_YS);

    const int half = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int j0 = half * DVB;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = a.T, H = a.H, DV = a.dv, N = a.N;

    if (threadIdx.x == 0) {
        for (int i = 0; i < B_NUM; ++i) mbar_init(&bar[i], (i == B_FULL0 || i == B_FULL1) ? 2 : 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, TM_COLS);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = *tmem_slot;

    if (warp == 0) {
        // ================================ producer ================================
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
        }
        int issued[2] = {0, 0}, v_issued = 0;
        for (int m = 0; m < N; ++m) {
            const int mc = REV ? N - 1 - m : m;  // chunk processed in iteration m
            const int s = m & 1, t0 = mc * C;
            // slot s and its factors are free once the preparation of chunk m-2 is done;
            // the chain's copy of k and its factors once the chain finished chunk m-2
            if (m >= 2 && !mbar_wait(&bar[B_EMPTY0 + s], ((m >> 1) - 1) & 1, abort_flag)) break;
            if (m >= 2 && !mbar_wait(&bar[B_KCFREE0 + s], ((m >> 1) - 1) & 1, abort_flag)) break;
            unsigned char *slot = sm + s * SLOT;
            if (lane == 0) {
                unsigned char *kc = sm + OFF_KC + s * 16384;
                mbar_arrive_tx(&bar[B_FULL0 + s], 6 * 8192);
                tma_load_4d(slot + 0, &tm_k, 0, h, t0, b, &bar[B_FULL0 + s]);
                tma_load_4d(slot + 8192, &tm_q, 0, h, t0, b, &bar[B_FULL0 + s]);
                tma_load_4d(slot + 16384, &tm_k, 64, h, t0, b, &bar[B_FULL0 + s]);
                tma_load_4d(slot + 24576, &tm_q, 64, h, t0, b, &bar[B_FULL0 + s]);
                tma_load_4d(kc, &tm_k, 0, h, t0, b, &bar[B_FULL0 + s]);
                tma_load_4d(kc + 8192, &tm_k, 64, h, t0, b, &bar[B_FULL0 + s]);
            }
            // in-chunk cumulative log gate and the row / column factors of this chunk
            {
                float lg[2], bt[2];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int t = t0 + lane + 32 * hh;
                    const size_t row = ((size_t)b * T + t) * H + h;
                    lg[hh] = 0.f;
                    bt[hh] = 0.f;
                    if (t < T) {
                        if (VAR == VAR_GATED) lg[hh] = tcf::bf(a.alpha, row);
                        bt[hh] = tcf::bf(a.beta, row);
                    }
                }
                float x0 = lg[0], x1 = lg[1];
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y0 = __shfl_up_sync(0xffffffffu, x0, o);
                    const float y1 = __shfl_up_sync(0xffffffffu, x1, o);
                    if (lane >= o) { x0 += y0; x1 += y1; }
                }
                x1 += __shfl_sync(0xffffffffu, x0, 31);
                const float gC = __shfl_sync(0xffffffffu, x1, 31);
                const float gm = __shfl_sync(0xffffffffu, x0, 31);
                float dev = fmaxf(fabsf(x0 - gm), fabsf(x1 - gm));
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) dev = fmaxf(dev, __shfl_xor_sync(0xffffffffu, dev, o));
                float *pf = pf_all + s * 448;
                const float xs[2] = {x0, x1};
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int r = lane + 32 * hh;
                    const float x = xs[hh], e = __expf(x), d = __expf(x - gm);
                    pf[PF_GC * 64 + r] = x;
                    pf[PF_ROWA * 64 + r] = bt[hh] * d;
                    pf[PF_ROWP * 64 + r] = d;
                    pf[PF_COLA * 64 + r] = __expf(gm - x);
                    pf[PF_BV * 64 + r] = bt[hh];
                    pf[PF_BK * 64 + r] = bt[hh] * e;
                    pf[PF_EG * 64 + r] = e;
                    cf[s * 80 + r] = __expf(gC - x);
                }
                if (lane == 0) {
                    cf[s * 80 + 64] = __expf(gC);
                    bigflag[s] = dev > 80.f;
                }
                if (SAVE && half == 0) {
                    float *Gc = a.G + (((size_t)b * H + h) * N + mc) * C;
                    Gc[lane] = xs[0];
                    Gc[lane + 32] = xs[1];
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[B_FULL0 + s]);
            issued[s]++;
            if (m >= 1 && !mbar_wait(&bar[B_VEMPTY], (m - 1) & 1, abort_flag)) break;
            if (lane == 0) {
                if (REV) {  // dO (and du) of this chunk for the chain
                    mbar_arrive_tx(&bar[B_VFULL], a.has_du ? 16384 : 8192);
                    tma_load_4d(sm + OFF_U, &tm_v, j0, h, t0, b, &bar[B_VFULL]);
                    if (a.has_du) tma_load_4d(sm + OFF_V, &tm_x, j0, h, t0, b, &bar[B_VFULL]);
                } else {
                    mbar_arrive_tx(&bar[B_VFULL], 8192);
                    tma_load_4d(sm + OFF_V, &tm_v, j0, h, t0, b, &bar[B_VFULL]);
                }
            }
            v_issued++;
        }
        if (*abort_flag) {
            volatile int dummy = 0;
            for (int s = 0; s < 2; ++s)
                if (issued[s] > 0) mbar_wait(&bar[B_FULL0 + s], (issued[s] - 1) & 1, &dummy, 100000000ull);
            if (v_issued > 0) mbar_wait(&bar[B_VFULL], (v_issued - 1) & 1, &dummy, 100000000ull);
        }
    } else if (warp <= 4) {
        // ============================ preparation warpgroup ============================
        const int wt = threadIdx.x - 32;
        const int q4 = warp & 3, trow = q4 * 32 + lane;
        const uint32_t tl = tbase + ((uint32_t)(q4 * 32) << 16);
        uint32_t ph = 0;
        bool pending = false;
        auto wsync = [&]() { named_sync(1, 128); };
        auto wabort = [&]() -> bool { return named_sync_any(1, 128, *abort_flag != 0); };
        auto mma_done = [&]() -> bool {
            mbar_wait(&bar[B_PMMA], ph & 1, abort_flag);
            ph++;
            fence_after_sync();
            const bool ok = !wabort();
            if (ok) pending = false;
            return ok;
        };
        float *Asc = reinterpret_cast<float *>(sm + OFF_RR);
        float *Tf = Asc + 4096;
        for (int m = 0; m < N; ++m) {
            const int mc = REV ? N - 1 - m : m;
            const int s = m & 1, bb = m & 1;
            unsigned char *slot = sm + s * SLOT;
            mbar_wait(&bar[B_FULL0 + s], (m >> 1) & 1, abort_flag);
            if (wabort()) break;
            const float *pf = pf_all + s * 448;
            if (REV) {  // the chain's copy of k becomes Kbar = e^{g_C - g} k
                unsigned char *kc = sm + OFF_KC + bb * 16384;
                const float *rowf = cf + bb * 80;
                for (int x = wt; x < 1024; x += 128) {
                    const int p = x >> 9, r = (x >> 3) & 63, ch = x & 7;
                    const uint32_t o = (uint32_t)p * 8192 + swz(r, ch);
                    float kv[8];
                    ld_chunk(kc, o, kv);
                    const float f = rowf[r];
#pragma unroll
                    for (int e = 0; e < 8; ++e) kv[e] *= f;
                    st_chunk(kc, o, kv);
                }
            }
            // ---------------- P1: [k ; q] . k^T ----------------
            if (wt == 0) {
                fence_after_sync();
                const uint32_t id = idesc_bf16(128, 64, 0, 0);
                const uint32_t sa = smem_u32(slot);
#pragma unroll
                for (int st = 0; st < 8; ++st) {
                    const uint32_t ad = sa + (st >> 2) * 16384 + (st & 3) * 32;
                    mma_bf16(tbase + TM_G1, sdesc(ad, 16, 1024), sdesc(ad, 16, 1024), id, st > 0);
                }
                mma_commit(&bar[B_PMMA]);
            }
            pending = true;
            if (!mma_done()) break;
            // ---------------- A, P, T ----------------
            {
                float g1[64];
                tmem_row64(tl + TM_G1, g1);
                const bool big = bigflag[s] != 0;
                const float *gc = pf + PF_GC * 64, *cola = pf + PF_COLA * 64;
                const bool arow = trow < 64;
                const int r = arow ? trow : trow - 64;
                // gate factor of each (r, i): e^{g_r - g_i}, split at the midpoint unless the range is large
                float f[64];
                if (VAR == VAR_DELTANET) {
#pragma unroll
                    for (int i = 0; i < 64; ++i) f[i] = 1.f;
                } else if (!big) {
                    const float4 *c4 = reinterpret_cast<const float4 *>(cola);
#pragma unroll
                    for (int i4 = 0; i4 < 16; ++i4) {
                        const float4 c = c4[i4];
                        f[4 * i4] = c.x; f[4 * i4 + 1] = c.y; f[4 * i4 + 2] = c.z; f[4 * i4 + 3] = c.w;
                    }
                    const float rf = pf[PF_ROWP * 64 + r];
#pragma unroll
                    for (int i = 0; i < 64; ++i) f[i] *= rf;
                } else {
                    const float gr = gc[r];
#pragma unroll
                    for (int i = 0; i < 64; ++i) f[i] = __expf(gr - gc[i]);
                }
                if (SAVE && arow && half == 0)
                    st_row_global(a.KK, ((((size_t)b * H + h) * N + mc) * C + r) * C, g1);
                if (arow) {
                    const float br = pf[PF_BV * 64 + r];
#pragma unroll
                    for (int i4 = 0; i4 < 16; ++i4) {
                        float4 v;
                        v.x = (4 * i4 + 0 < r) ? g1[4 * i4 + 0] * f[4 * i4 + 0] * br : 0.f;
                        v.y = (4 * i4 + 1 < r) ? g1[4 * i4 + 1] * f[4 * i4 + 1] * br : 0.f;
                        v.z = (4 * i4 + 2 < r) ? g1[4 * i4 + 2] * f[4 * i4 + 2] * br : 0.f;
                        v.w = (4 * i4 + 3 < r) ? g1[4 * i4 + 3] * f[4 * i4 + 3] * br : 0.f;
                        *reinterpret_cast<float4 *>(&Asc[sw64(r, 4 * i4)]) = v;
                    }
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        float w[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) w[e] = (ch * 8 + e == r) ? 1.f : 0.f;
                        st_chunk(sm + OFF_IP, swz(r, ch), w);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 64; ++i) g1[i] = (i <= r) ? g1[i] * f[i] : 0.f;
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) st_chunk(sm + OFF_IP, swz(trow, ch), g1 + ch * 8);
                    if (SAVE && half == 0) st_row_global(a.P, ((((size_t)b * H + h) * N + mc) * C + r) * C, g1);
                }
                fence_before_sync();
                wsync();
                unit_lower_inverse64(Asc, Tf, ysc, wt, wsync);
                if (wt < 64) {
                    const int i = wt;
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        const float4 lo = *reinterpret_cast<const float4 *>(&Tf[sw64(i, ch * 8)]);
                        const float4 hi = *reinterpret_cast<const float4 *>(&Tf[sw64(i, ch * 8 + 4)]);
                        float w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
                        for (int e = 0; e < 8; ++e) w[e] = (ch * 8 + e <= i) ? w[e] : 0.f;
                        st_chunk(sm + OFF_TT, swz(i, ch), w);
                        if (SAVE && half == 0)
                            st8_global(a.Tn, ((((size_t)b * H + h) * N + mc) * C + i) * C + ch * 8, w);
                    }
                }
                fence_proxy_async();
                wsync();
            }
            // ---------------- IPT: R = [I ; P] T ----------------
            if (wt == 0) {
                fence_after_sync();
                const uint32_t id = idesc_bf16(128, 64, 0, 1);
                const uint32_t ip = smem_u32(sm + OFF_IP), tt = smem_u32(sm + OFF_TT);
#pragma unroll
                for (int st = 0; st < 4; ++st)
                    mma_bf16(tbase + TM_G1, sdesc(ip + st * 32, 16, 1024), sdesc(tt + st * 2048, 1024, 1024), id,
                             st > 0);
                mma_commit(&bar[B_PMMA]);
            }
            pending = true;
            if (!mma_done()) break;
            // ---------------- R diag(beta), R diag(beta e^g) ----------------
            {
                float rv[64];
                tmem_row64(tl + TM_G1, rv);
                const float *bv = pf + PF_BV * 64, *bk = pf + PF_BK * 64;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    float w[8], w2[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        w[e] = rv[ch * 8 + e] * bv[ch * 8 + e];
                        w2[e] = rv[ch * 8 + e] * bk[ch * 8 + e];
                    }
                    st_chunk(sm + OFF_RR, swz(trow, ch), w);
                    st_chunk(sm + OFF_RR + 16384, swz(trow, ch), w2);
                }
            }
            if (!REV) {
                mbar_wait(&bar[B_VFULL], m & 1, abort_flag);
                if (m >= 2) mbar_wait(&bar[B_DFREE0 + bb], ((m >> 1) - 1) & 1, abort_flag);
            }
            fence_proxy_async();
            fence_before_sync();
            if (wabort()) break;
            // ---------------- P3: X = [W ; P W];  P4: D = [U~ ; P U~] ----------------
            if (wt == 0) {
                fence_after_sync();
                const uint32_t rr = smem_u32(sm + OFF_RR), sk = smem_u32(slot), vv = smem_u32(sm + OFF_V);
                const uint32_t id3 = idesc_bf16(128, 128, 0, 1), id4 = idesc_bf16(128, 64, 0, 1);
#pragma unroll
                for (int st = 0; st < 4; ++st)
                    mma_bf16(tbase + TM_X, sdesc(rr + 16384 + st * 32, 16, 1024), sdesc(sk + st * 2048, 16384, 1024),
                             id3, st > 0);
                if (!REV) {
#pragma unroll
                    for (int st = 0; st < 4; ++st)
                        mma_bf16(tbase + TM_D0 + bb * 64, sdesc(rr + st * 32, 16, 1024),
                                 sdesc(vv + st * 2048, 1024, 1024), id4, st > 0);
                }
                mma_commit(&bar[B_PMMA]);
            }
            pending = true;
            if (!mma_done()) break;
            if (!REV && wt == 0) mbar_arrive(&bar[B_VEMPTY]);
            if (SAVE && trow < 64) {
                const size_t ci = ((size_t)b * H + h) * N + mc;
                float rv[64];
                tmem_row64(tl + TM_D0 + bb * 64, rv);
                st_row_global(a.Ut, (ci * C + trow) * DV + j0, rv);
                if (half == 0) {
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        tmem_row64(tl + TM_X + hh * 64, rv);
                        st_row_global(a.W, (ci * C + trow) * DK + hh * 64, rv);
                    }
                }
            }
            // ---------------- A_chain ----------------
            if (m >= 1) mbar_wait(&bar[B_ACFREE], (m - 1) & 1, abort_flag);
            if (wabort()) break;
            {
                const int r = trow;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float xv[64];
                    tmem_row64(tl + TM_X + hh * 64, xv);
                    if (r < 64) {
#pragma unroll
                        for (int i = 0; i < 64; ++i) xv[i] = -xv[i];
                    } else {
                        const int rr = r - 64;
                        const float sc = pf[PF_EG * 64 + rr];
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch) {
                            float qv[8];
                            ld_chunk(slot, (uint32_t)hh * 16384 + 8192 + swz(rr, ch), qv);
#pragma unroll
                            for (int e = 0; e < 8; ++e) xv[ch * 8 + e] = qv[e] * sc - xv[ch * 8 + e];
                        }
                    }
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) st_chunk(sm + OFF_AC, (uint32_t)hh * 16384 + swz(r, ch), xv + ch * 8);
                }
            }
            fence_proxy_async();
            fence_before_sync();
            wsync();
            if (wt == 0) {
                mbar_arrive(&bar[B_EMPTY0 + s]);
                mbar_arrive(&bar[B_READY0 + bb]);
            }
        }
        if (*abort_flag && pending) {
            volatile int dummy = 0;
            mbar_wait(&bar[B_PMMA], ph & 1, &dummy, 100000000ull);
        }
    } else {
        // ================================ chain warpgroup ================================
        const int wc = threadIdx.x - 160;
        const int q4 = warp & 3, trow = q4 * 32 + lane;
        const uint32_t tl = tbase + ((uint32_t)(q4 * 32) << 16);
        uint32_t ph = 0;
        bool pending = false;
        auto wsync = [&]() { named_sync(2, 128); };
        auto wabort = [&]() -> bool { return named_sync_any(2, 128, *abort_flag != 0); };
        auto mma_done = [&]() -> bool {
            mbar_wait(&bar[B_CMMA], ph & 1, abort_flag);
            ph++;
            fence_after_sync();
            const bool ok = !wabort();
            if (ok) pending = false;
            return ok;
        };
        float S[DVB];
        {
            const float *s0 = a.S0 ? a.S0 + (((size_t)b * H + h) * DK + trow) * DV + j0 : nullptr;
#pragma unroll
            for (int j = 0; j < DVB; ++j) S[j] = s0 ? s0[j] : 0.f;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) st_chunk(sm + OFF_S, swz(trow, ch), S + ch * 8);
        }
        fence_proxy_async();
        wsync();
        if (REV) {
            // ---------------- reverse chain: S holds dS of the state leaving chunk mc ----------------
            for (int m = 0; m < N; ++m) {
                const int mc = N - 1 - m, bb = m & 1;
                mbar_wait(&bar[B_READY0 + bb], (m >> 1) & 1, abort_flag);
                mbar_wait(&bar[B_VFULL], m & 1, abort_flag);
                if (wabort()) break;
                st_row_global(a.dSn, ((((size_t)b * H + h) * N + mc) * DK + trow) * DV + j0, S);
                // G = (-W)^T Kbar  and  D = A_chain^T [du ; dO]
                if (wc == 0) {
                    fence_after_sync();
                    const uint32_t ac = smem_u32(sm + OFF_AC), kc = smem_u32(sm + OFF_KC + bb * 16384);
                    const uint32_t dub = smem_u32(sm + OFF_V), dob = smem_u32(sm + OFF_U);
                    const uint32_t idg = idesc_bf16(128, 128, 1, 1), idd = idesc_bf16(128, 64, 1, 1);
#pragma unroll
                    for (int st = 0; st < 4; ++st)
                        mma_bf16(tbase + TM_G, sdesc(ac + st * 2048, 16384, 1024), sdesc(kc + st * 2048, 8192, 1024), idg,
                                 st > 0);
                    const int st0 = a.has_du ? 0 : 4;
                    for (int st = st0; st < 8; ++st) {
                        const uint32_t bsrc = st < 4 ? dub + st * 2048 : dob + (st - 4) * 2048;
                        mma_bf16(tbase + TM_D0 + bb * 64, sdesc(ac + st * 2048, 16384, 1024), sdesc(bsrc, 1024, 1024),
                                 idd, st > st0);
                    }
                    mma_commit(&bar[B_CMMA]);
                }
                pending = true;
                if (!mma_done()) break;
                if (wc == 0) mbar_arrive(&bar[B_VEMPTY]);
                // M' = G -> bf16, K-major A operand in the A_chain region (A_chain is consumed)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float gv[64];
                    tmem_row64(tl + TM_G + hh * 64, gv);
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) st_chunk(sm + OFF_AC, (uint32_t)hh * 16384 + swz(trow, ch), gv + ch * 8);
                }
                fence_proxy_async();
                fence_before_sync();
                wsync();
                // D += M' dS+
                if (wc == 0) {
                    fence_after_sync();
                    const uint32_t ac = smem_u32(sm + OFF_AC), ss = smem_u32(sm + OFF_S);
                    const uint32_t id = idesc_bf16(128, 64, 0, 1);
#pragma unroll
                    for (int st = 0; st < 8; ++st)
                        mma_bf16(tbase + TM_D0 + bb * 64, sdesc(ac + (st >> 2) * 16384 + (st & 3) * 32, 16, 1024),
                                 sdesc(ss + st * 2048, 1024, 1024), id, 1);
                    mma_commit(&bar[B_CMMA]);
                }
                pending = true;
                if (!mma_done()) break;
                if (wc == 0) mbar_arrive(&bar[B_ACFREE]);
                {
                    float dv[64];
                    tmem_row64(tl + TM_D0 + bb * 64, dv);
                    const float gmc = cf[bb * 80 + 64];
#pragma unroll
                    for (int j = 0; j < DVB; ++j) S[j] = gmc * S[j] + dv[j];
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) st_chunk(sm + OFF_S, swz(trow, ch), S + ch * 8);
                }
                fence_proxy_async();
                fence_before_sync();
                wsync();
                if (wc == 0) mbar_arrive(&bar[B_KCFREE0 + bb]);
            }
        } else
        for (int m = 0; m < N; ++m) {
            const int bb = m & 1, t0 = m * C;
            const int L = min(C, T - t0);
            mbar_wait(&bar[B_READY0 + bb], (m >> 1) & 1, abort_flag);
            if (wabort()) break;
            if (SAVE) st_row_global(a.Sn, ((((size_t)b * H + h) * N + m) * DK + trow) * DV + j0, S);
            // ---------------- C1: D += A_chain . S ----------------
            if (wc == 0) {
                fence_after_sync();
                const uint32_t id = idesc_bf16(128, 64, 0, 1);
                const uint32_t ac = smem_u32(sm + OFF_AC), ss = smem_u32(sm + OFF_S);
#pragma unroll
                for (int st = 0; st < 8; ++st)
                    mma_bf16(tbase + TM_D0 + bb * 64, sdesc(ac + (st >> 2) * 16384 + (st & 3) * 32, 16, 1024),
                             sdesc(ss + st * 2048, 1024, 1024), id, 1);
                mma_commit(&bar[B_CMMA]);
            }
            pending = true;
            if (!mma_done()) break;
            if (wc == 0) mbar_arrive(&bar[B_ACFREE]);
            // ---------------- write values and outputs ----------------
            {
                float dv[64];
                tmem_row64(tl + TM_D0 + bb * 64, dv);
                if (trow < 64) {
                    const int r = trow;
                    if (SAVE) st_row_global(a.Un, ((((size_t)b * H + h) * N + m) * C + r) * DV + j0, dv);
                    else if (a.u && r < L) {
                        st_row_global(a.u, (((size_t)b * T + t0 + r) * H + h) * DV + j0, dv);
                    }
                    const float f = cf[bb * 80 + r];
#pragma unroll
                    for (int i = 0; i < 64; ++i) dv[i] *= f;
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) st_chunk(sm + OFF_U, swz(r, ch), dv + ch * 8);
                } else {
                    const int r = trow - 64;
                    if (!SAVE && r < L) st_row_global(a.out, (((size_t)b * T + t0 + r) * H + h) * DV + j0, dv);
                }
            }
            fence_proxy_async();
            fence_before_sync();
            wsync();
            if (wc == 0) mbar_arrive(&bar[B_DFREE0 + bb]);
            // ---------------- C3: E = k^T (e^{gC-g} U) ----------------
            if (wc == 0) {
                fence_after_sync();
                const uint32_t id = idesc_bf16(128, 64, 1, 1);
                const uint32_t kc = smem_u32(sm + OFF_KC + bb * 16384), uu = smem_u32(sm + OFF_U);
#pragma unroll
                for (int st = 0; st < 4; ++st)
                    mma_bf16(tbase + TM_E, sdesc(kc + st * 2048, 8192, 1024), sdesc(uu + st * 2048, 1024, 1024), id,
                             st > 0);
                mma_commit(&bar[B_CMMA]);
            }
            pending = true;
            if (!mma_done()) break;
            // ---------------- S <- e^{gC} S + E ----------------
            {
                float ev[64];
                tmem_row64(tl + TM_E, ev);
                const float gmc = cf[bb * 80 + 64];
#pragma unroll
                for (int j = 0; j < DVB; ++j) S[j] = gmc * S[j] + ev[j];
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) st_chunk(sm + OFF_S, swz(trow, ch), S + ch * 8);
            }
            fence_proxy_async();
            fence_before_sync();
            wsync();
            if (wc == 0) mbar_arrive(&bar[B_KCFREE0 + bb]);
        }
        if (*abort_flag == 0) {
            if (MODE != 1 && a.ST) {
                float *dst = a.ST + (((size_t)b * H + h) * DK + trow) * DV + j0;
#pragma unroll
                for (int j = 0; j < DVB; j += 4)
                    *reinterpret_cast<float4 *>(dst + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
            }
        } else if (pending) {
            volatile int dummy = 0;
            mbar_wait(&bar[B_CMMA], ph & 1, &dummy, 100000000ull);
        }
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == 0) tmem_dealloc(tbase, TM_COLS);
}

}  // namespace tcf2

template <int VAR, int MODE>
static cudaError_t launch_tc2(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                              const CUtensorMap &mx, const tcf2::Args &a, dim3 grid, size_t smem, cudaStream_t s,
                              Rec &rec) {
    cudaError_t e = cudaFuncSetAttribute(tcf2::k_fwd_tc2<VAR, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    rec.mark(s);
    tcf2::k_fwd_tc2<VAR, MODE><<<grid, tcf2::NTHREADS, smem, s>>>(mq, mk, mv, mx, a);
    return cudaGetLastError();
}

static cudaError_t tc2_common(const Geo &g, const Tensors &t, const TcBwdWs *w, int mode, cudaStream_t s, Rec &rec) {
    using namespace tcf2;
    CUtensorMap mq, mk, mv, mx;
    const uint64_t Bn = g.B, T = g.T, H = g.H;
    const void *vsrc = mode == 2 ? t.dout : t.v;
    bool ok = tc::make_map_4d_bf16(&mq, t.q, DK, H, T, Bn, 64) && tc::make_map_4d_bf16(&mk, t.k, DK, H, T, Bn, 64) &&
              tc::make_map_4d_bf16(&mv, vsrc, g.dv, H, T, Bn, 64);
    if (ok && mode == 2 && t.du) ok = tc::make_map_4d_bf16(&mx, t.du, g.dv, H, T, Bn, 64);
    else mx = mv;
    if (!ok) return cudaErrorInvalidValue;
    Args a = {};
    a.alpha = t.alpha; a.beta = t.beta; a.B = g.B; a.T = g.T; a.H = g.H; a.dv = g.dv; a.N = g.N;
    if (mode == 2) {
        a.S0 = t.dS_T; a.ST = t.dS0; a.dSn = w->dSn; a.has_du = t.du != nullptr;
    } else {
        a.S0 = t.S0; a.out = t.out; a.u = t.u; a.ST = t.S_T;
    }
    if (mode == 1) {
        a.W = w->W; a.Ut = w->Ut; a.G = w->g; a.P = w->P; a.Sn = w->Sn; a.Un = w->Un;
        a.Tn = w->Tn; a.KK = w->KK;
    }
    const dim3 grid(g.dv / DVB, g.H, g.B);
    const size_t smem = SMEM_BYTES + 1024;
    if (g.variant == VAR_GATED) {
        if (mode == 0) return launch_tc2<VAR_GATED, 0>(mq, mk, mv, mx, a, grid, smem, s, rec);
        if (mode == 1) return launch_tc2<VAR_GATED, 1>(mq, mk, mv, mx, a, grid, smem, s, rec);
        return launch_tc2<VAR_GATED, 2>(mq, mk, mv, mx, a, grid, smem, s, rec);
    }
    if (mode == 0) return launch_tc2<VAR_DELTANET, 0>(mq, mk, mv, mx, a, grid, smem, s, rec);
    if (mode == 1) return launch_tc2<VAR_DELTANET, 1>(mq, mk, mv, mx, a, grid, smem, s, rec);
    return launch_tc2<VAR_DELTANET, 2>(mq, mk, mv, mx, a, grid, smem, s, rec);
}

// Warp-specialised forward (Gated DeltaNet / DeltaNet).
cudaError_t tc_fwd2(const Geo &g, const Tensors &t, cudaStream_t s, Rec &rec) { return tc2_common(g, t, nullptr, 0, s, rec); }

// The same kernel in recompute mode: fills g, KK, P, T, W, U~, S_n, U of the backward workspace.
cudaError_t tc_bwd_recompute(const Geo &g, const Tensors &t, const TcBwdWs &w, cudaStream_t s, Rec &rec) {
    return tc2_common(g, t, &w, 1, s, rec);
}

// The same kernel in reverse mode: fills dS_{n+1} of every chunk and writes dS0.
cudaError_t tc_bwd_reverse(const Geo &g, const Tensors &t, const TcBwdWs &w, cudaStream_t s, Rec &rec) {
    return tc2_common(g, t, &w, 2, s, rec);
}

}  // namespace dr
