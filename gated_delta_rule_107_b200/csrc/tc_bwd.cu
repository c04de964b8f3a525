// tc_bwd.cu -- all intra-chunk gradients of the backward on tcgen05 (Gated DeltaNet, DeltaNet).
//
// Backward of the chunked form of "线性注意力架构演进与Kimi Delta Attention创新实践"
// (sections 2.1, 6.2, 7.1) for one chunk of one (b, h), scalar gates.  With g the in-chunk
// cumulative log gate, E_ri = e^{g_r - g_i} (i <= r), S = S_n, dS+ = dL/dS_{n+1} (from the
// reverse chain), and W, U~, U, P, T = (I+A)^-1, KK = k k^T, A = diag(beta) (KK .* E) saved by
// the recompute:
//
//   dU   = du + P^T dO + Kbar dS+              Kbar = e^{g_C - g} k
//   dP   = tril(dO U^T)                        dW = -dU S^T
//   dB_k = T^T dW,  dB_v = T^T dU              (through W = T diag(beta e^g) k, U~ = T diag(beta) v)
//   dA   = -strict_tril(dB_k W^T + dB_v U~^T)
//   D_P  = dP .* E,  D_M = diag(beta) dA .* E
//   dq   = diag(e^g) dO S^T + D_P k
//   dk   = D_P^T q + (D_M + D_M^T) k + diag(beta e^g) dB_k + diag(e^{g_C - g}) U dS+^T
//   dv   = diag(beta) dB_v
//   dbeta_r = (dA .* KK .* E)_r. + e^{g_r} k_r . dB_k,r + v_r . dB_v,r
//   dg_r = e^{g_r} q_r . (dO S^T)_r + rowsum_r(Z) - colsum_r(Z) + beta_r e^{g_r} k_r . dB_k,r
//          - e^{g_C - g_r} k_r . (U dS+^T)_r,   Z = dP .* P + dA .* A,
//   dg_C += sum_r e^{g_C - g_r} k_r . (U dS+^T)_r + e^{g_C} sum(S .* dS+);
//   d log alpha = reverse cumulative sum of dg over the chunk.
//
// The dense products run channel-major so that M = 128 (dk or dv) fills the MMA; the two
// token x token products (dP, dA) use M = 128 MMAs whose rows 64..127 read other (valid)
// shared memory and are discarded.  D_M + D_M^T needs no transpose: the same D_M tile is
// read once as an MN-major and once as a K-major B operand.
//
// One CTA of 256 threads per chunk.  Every operand tile arrives by TMA in two groups: what
// the first products read (S, dS+, U, dO, k, P, T, KK, du), then -- once those products
// have consumed their inputs -- W, U~, q, k, v into the space they freed.  dq, dk and dv
// leave through shared-memory staging tiles and TMA stores.  Warps w and w + 4 read the
// same 32 TMEM lanes (channel rows) and split the 64 token columns; sums over channels
// are butterfly transposes inside a warp plus four partials in shared memory.
#include "tc_host.cuh"
#include "tc_path.cuh"
#include "tc_ptx.cuh"
#include "tc_tile.cuh"

namespace dr {
namespace tcb {

using namespace dr::tc;
using dr::tcf::ld_chunk;
using dr::tcf::st_chunk;
using dr::tcf::tok_off;

constexpr int C = 64, DK = 128, DV = 128;
constexpr int NTHREADS = 256;
// shared memory (bytes from a 1024-aligned base); later phases reuse earlier regions
constexpr uint32_t R_S = 0;          // 32K  S [c][j]     -> dB_k^T [c][i] (16K) | dB_v^T [j][i] (16K)
constexpr uint32_t R_DS = 32768;     // 32K  dS+ [c][j]   -> W [i][c] | U~ [i][j]  -> dk staging [r][c]
constexpr uint32_t R_U = 65536;      // 16K  U [r][j]     -> q [r][c]
constexpr uint32_t R_DO = 81920;     // 16K  dO [r][j]    -> k [r][c]
constexpr uint32_t R_KB = 98304;     // 16K  Kbar [r][c]  -> v [r][j]
constexpr uint32_t R_P = 114688;     //  8K  P [r][i]     -> D_P [r][i]
constexpr uint32_t R_T = 122880;     //  8K  T [r][i]     -> D_M [r][i]
constexpr uint32_t R_KK = 131072;    //  8K  KK [r][i]
constexpr uint32_t R_DU = 139264;    // 16K  du [r][j]
constexpr uint32_t R_DUT = 155648;   // 16K  dU^T [j][r]  -> dv staging [i][j]
constexpr uint32_t R_DWT = 172032;   // 16K  dW^T [c][r]  -> dq staging [r][c]
constexpr uint32_t R_MISC = 188416;  //  8K
constexpr uint32_t SMEM_BYTES = R_MISC + 8192;
// bytes of the two TMA load groups
constexpr uint32_t LOAD1_BYTES = 2 * 32768 + 3 * 16384 + 3 * 8192;  // + du (16K) when given
constexpr uint32_t LOAD2_BYTES = 5 * 16384;
// misc (floats unless noted)
constexpr uint32_t M_BAR = 0;  // [0] MMA batches, [1] first load group, [2] second load group
constexpr uint32_t M_TMEM = 64, M_ABORT = 68;
constexpr uint32_t M_GC = 256, M_BETA = 512, M_EG = 768, M_EGC = 1024;  // [64] each
constexpr uint32_t M_RED = 1280;                    // [5 kinds][4 lane quarters][64 tokens]
constexpr uint32_t M_ROW = M_RED + 5 * 4 * 64 * 4;  // [2 column halves][64] rowsum Z, then [2][64] dbeta (A part)
constexpr uint32_t M_RS = M_ROW + 4 * 64 * 4;       // [8 warps] partial sums of S .* dS+
constexpr uint32_t M_DG = M_RS + 64;                // [64] dg, then [64] the k . Tm sums
static_assert(M_DG + 512 <= 8192, "misc overflow");
enum { RK_QQD = 0, RK_KBK, RK_KTM, RK_VBV, RK_ZC };
// TMEM columns
constexpr uint32_t TM_DUT = 0, TM_QD = 64, TM_TM = 128, TM_DP = 192, TM_DW = 256, TM_DBK = 320, TM_DQ = 384,
                   TM_DK = 448, TM_COLS = 512;

struct Maps {
    CUtensorMap q, k, v, dout, du, dq, dk, dv;  // [B, T, H, 128] bf16; box 64 channels x 64 tokens
    CUtensorMap S, dS;                          // [chunks * 128][128] bf16; box 64 x 128
    CUtensorMap U, W, Ut;                       // [chunks * 64][128] bf16; box 64 x 64
    CUtensorMap P, T, KK;                       // [chunks * 64][64] bf16; box 64 x 64
};

struct Args {
    const void *beta;        // bf16 [B, T, H]
    void *dalpha, *dbeta;    // bf16 [B, T, H]
    const float *g;          // [chunks][64]
    int B, T, H, N, variant, has_du;
};

__device__ __forceinline__ void st_bf(void *p, size_t i, float x) {
    reinterpret_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(x);
}
__device__ __forceinline__ float ld_tile(const unsigned char *base, int r, int c) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(base + tok_off(r, c)));
}
__device__ __forceinline__ void st_tile(unsigned char *base, int r, int c, float x) {
    *reinterpret_cast<__nv_bfloat16 *>(base + tok_off(r, c)) = __float2bfloat16_rn(x);
}

// 32 fp32 columns of this thread's TMEM lane
__device__ __forceinline__ void tmem_row32(uint32_t taddr, float *v) {
    tmem_ld16(taddr + 0, v);
    tmem_ld16(taddr + 16, v + 16);
    wait_ld();
}

// v[t] (t = 0..31) held by every lane of the warp; returns sum over the 32 lanes of v[lane].
// Butterfly transpose: at each step a lane keeps half of its live values and adds the
// partner's copy of that half (16 + 8 + 4 + 2 + 1 shuffles).
__device__ __forceinline__ float warp_colsum32(float *v, int lane) {
#pragma unroll
    for (int s = 0; s < 5; ++s) {
        const int m = 16 >> s;
        const bool up = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < m; ++i) {
            const float lo = v[i], hi = v[i + m];
            const float send = up ? lo : hi;
            v[i] = (up ? hi : lo) + __shfl_xor_sync(0xffffffffu, send, m);
        }
    }
    return v[0];
}

__global__ void __launch_bounds__(NTHREADS, 1) k_bwd_chunk_tc(const __grid_constant__ Maps mp, Args a) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + R_MISC + M_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + R_MISC + M_TMEM);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + R_MISC + M_ABORT);
    float *gc = reinterpret_cast<float *>(sm + R_MISC + M_GC);
    float *betas = reinterpret_cast<float *>(sm + R_MISC + M_BETA);
    float *eg = reinterpret_cast<float *>(sm + R_MISC + M_EG);
    float *egc = reinterpret_cast<float *>(sm + R_MISC + M_EGC);
    float *red = reinterpret_cast<float *>(sm + R_MISC + M_RED);
    float *rowsum = reinterpret_cast<float *>(sm + R_MISC + M_ROW);
    float *rsp = reinterpret_cast<float *>(sm + R_MISC + M_RS);
    float *dgs = reinterpret_cast<float *>(sm + R_MISC + M_DG);
    float *ktm = dgs + 64;

    const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, hf = warp >> 2;
    const int lr = quarter * 32 + lane;  // TMEM lane: channel row of the channel-major products
    const int col0 = hf * 32;            // first of this thread's 32 token columns
    const int T = a.T, H = a.H, t0 = n * C, L = min(C, T - t0);
    const int ci = (b * H + h) * a.N + n;  // < 2^31 / 128 (checked by the launcher)
    const bool gated = a.variant == VAR_GATED;
    auto trow_g = [&](int r) -> size_t { return ((size_t)b * T + t0 + r) * H + h; };  // token row (r < L)
    auto red_at = [&](int kind, int q, int t) -> float & { return red[(kind * 4 + q) * 64 + t]; };

    // issue state of thread 0 (the only thread that issues TMA and MMA)
    int mma_issued = 0, loads_issued = 0;
    if (tid == 0) {
        for (int i = 0; i < 3; ++i) mbar_init(&bar[i], 1);
        *abort_flag = 0;
        fence_mbar_init();
        mbar_arrive_tx(&bar[1], LOAD1_BYTES + (a.has_du ? 16384u : 0u));
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            tma_load_2d(sm + R_S + p * 16384, &mp.S, 64 * p, ci * DK, &bar[1]);
            tma_load_2d(sm + R_DS + p * 16384, &mp.dS, 64 * p, ci * DK, &bar[1]);
            tma_load_2d(sm + R_U + p * 8192, &mp.U, 64 * p, ci * C, &bar[1]);
            tma_load_4d(sm + R_DO + p * 8192, &mp.dout, 64 * p, h, t0, b, &bar[1]);
            tma_load_4d(sm + R_KB + p * 8192, &mp.k, 64 * p, h, t0, b, &bar[1]);
            if (a.has_du) tma_load_4d(sm + R_DU + p * 8192, &mp.du, 64 * p, h, t0, b, &bar[1]);
        }
        tma_load_2d(sm + R_P, &mp.P, 0, ci * C, &bar[1]);
        tma_load_2d(sm + R_T, &mp.T, 0, ci * C, &bar[1]);
        tma_load_2d(sm + R_KK, &mp.KK, 0, ci * C, &bar[1]);
        loads_issued = 1;
    }
    if (warp == 0) tmem_alloc(tmem_slot, TM_COLS);
    if (tid < C) {
        const float x = a.g[(size_t)ci * C + tid];
        gc[tid] = x;
        betas[tid] = (tid < L) ? tcf::bf(a.beta, trow_g(tid)) : 0.f;
        eg[tid] = __expf(x);
        egc[tid] = __expf(a.g[(size_t)ci * C + C - 1] - x);
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tl = tbase + ((uint32_t)(quarter * 32) << 16) + (uint32_t)col0;
    uint32_t ph = 0;
    auto consensus = [&](bool ok) -> bool { return !named_sync_any(1, NTHREADS, !ok || *abort_flag != 0); };
    auto wait_mma = [&]() -> bool {
        const bool ok = mbar_wait(&bar[0], ph & 1, abort_flag);
        ph++;
        fence_after_sync();
        return consensus(ok);
    };
    const uint32_t sS = smem_u32(sm + R_S), sD = smem_u32(sm + R_DS), sU = smem_u32(sm + R_U);
    const uint32_t sO = smem_u32(sm + R_DO), sK = smem_u32(sm + R_KB), sP = smem_u32(sm + R_P);
    const uint32_t sT = smem_u32(sm + R_T), sUT = smem_u32(sm + R_DUT), sWT = smem_u32(sm + R_DWT);

    // ---------------- phase 0: Kbar = e^{g_C - g} k in place; sum of S .* dS+ ----------------
    bool ok = mbar_wait(&bar[1], 0, abort_flag);
    if (ok) {
        for (int x = tid; x < 1024; x += NTHREADS) {  // 2 panels x 64 rows x 8 chunks of 16 B
            float v[8];
            ld_chunk(sm + R_KB, (uint32_t)x * 16, v);
            const float f = egc[(x >> 3) & 63];
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] *= f;
            st_chunk(sm + R_KB, (uint32_t)x * 16, v);
        }
        float rs = 0.f;
        for (int x = tid; x < 2048; x += NTHREADS) {  // S and dS+ share one layout
            float v[8], w[8];
            ld_chunk(sm + R_S, (uint32_t)x * 16, v);
            ld_chunk(sm + R_DS, (uint32_t)x * 16, w);
#pragma unroll
            for (int e = 0; e < 8; ++e) rs += v[e] * w[e];
        }
        rs = warp_sum(rs);
        if (lane == 0) rsp[warp] = rs;
    }
    fence_proxy_async();
    fence_before_sync();
    ok = consensus(ok);

    // ---------------- batch 1: dU^T, Qd^T, Tm^T, dP ----------------
    if (ok && tid == 0) {
        fence_after_sync();
        const uint32_t id_mm = idesc_bf16(128, 64, 1, 1), id_mk = idesc_bf16(128, 64, 1, 0);
        const uint32_t id_kk = idesc_bf16(128, 64, 0, 0);
#pragma unroll
        for (int st = 0; st < 4; ++st)  // dO^T P
            mma_bf16(tbase + TM_DUT, sdesc(sO + st * 2048, 8192, 1024), sdesc(sP + st * 2048, 1024, 1024), id_mm,
                     st > 0);
#pragma unroll
        for (int st = 0; st < 8; ++st)  // + dS+^T Kbar^T
            mma_bf16(tbase + TM_DUT, sdesc(sD + st * 2048, 16384, 1024),
                     sdesc(sK + (st >> 2) * 8192 + (st & 3) * 32, 16, 1024), id_mk, 1);
#pragma unroll
        for (int st = 0; st < 8; ++st) {
            const uint32_t ka = (st >> 2) * 16384 + (st & 3) * 32, kb = (st >> 2) * 8192 + (st & 3) * 32;
            mma_bf16(tbase + TM_QD, sdesc(sS + ka, 16, 1024), sdesc(sO + kb, 16, 1024), id_kk, st > 0);  // S dO^T
            mma_bf16(tbase + TM_TM, sdesc(sD + ka, 16, 1024), sdesc(sU + kb, 16, 1024), id_kk, st > 0);  // dS+ U^T
            mma_bf16(tbase + TM_DP, sdesc(sO + kb, 16, 1024), sdesc(sU + kb, 16, 1024), id_kk, st > 0);  // dO U^T
        }
        mma_commit(&bar[0]);
        mma_issued++;
    }
    if (ok) ok = wait_mma();
    // second load group into the regions batch 1 has finished reading
    if (ok && tid == 0) {
        mbar_arrive_tx(&bar[2], LOAD2_BYTES);
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            tma_load_2d(sm + R_DS + p * 8192, &mp.W, 64 * p, ci * C, &bar[2]);
            tma_load_2d(sm + R_DS + 16384 + p * 8192, &mp.Ut, 64 * p, ci * C, &bar[2]);
            tma_load_4d(sm + R_U + p * 8192, &mp.q, 64 * p, h, t0, b, &bar[2]);
            tma_load_4d(sm + R_DO + p * 8192, &mp.k, 64 * p, h, t0, b, &bar[2]);
            tma_load_4d(sm + R_KB + p * 8192, &mp.v, 64 * p, h, t0, b, &bar[2]);
        }
        loads_issued = 2;
    }
    // ---------------- epilogue 1: dU (+ du) -> dU^T tile ----------------
    if (ok) {
        float v[32];
        tmem_row32(tl + TM_DUT, v);
        const int j = lr;
        if (a.has_du) {
#pragma unroll
            for (int t = 0; t < 32; ++t) v[t] += ld_tile(sm + R_DU, col0 + t, j);
        }
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) st_chunk(sm + R_DUT, swz(j, hf * 4 + c4), v + c4 * 8);
    }
    fence_proxy_async();
    fence_before_sync();
    ok = consensus(ok);
    // ---------------- batch 2: dW^T = -S dU^T ----------------
    if (ok && tid == 0) {
        fence_after_sync();
        const uint32_t id = idesc_bf16(128, 64, 0, 1, 1);
#pragma unroll
        for (int st = 0; st < 8; ++st)
            mma_bf16(tbase + TM_DW, sdesc(sS + (st >> 2) * 16384 + (st & 3) * 32, 16, 1024),
                     sdesc(sUT + st * 2048, 1024, 1024), id, st > 0);
        mma_commit(&bar[0]);
        mma_issued++;
    }
    if (ok) ok = wait_mma();
    if (ok) {
        float v[32];
        tmem_row32(tl + TM_DW, v);
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) st_chunk(sm + R_DWT, swz(lr, hf * 4 + c4), v + c4 * 8);
    }
    fence_proxy_async();
    fence_before_sync();
    ok = consensus(ok);
    // ---------------- batch 3: dB_k^T = dW^T T, dB_v^T = dU^T T ----------------
    if (ok && tid == 0) {
        fence_after_sync();
        const uint32_t id = idesc_bf16(128, 64, 0, 1);
#pragma unroll
        for (int st = 0; st < 4; ++st) {
            mma_bf16(tbase + TM_DBK, sdesc(sWT + st * 32, 16, 1024), sdesc(sT + st * 2048, 1024, 1024), id, st > 0);
            mma_bf16(tbase + TM_DUT, sdesc(sUT + st * 32, 16, 1024), sdesc(sT + st * 2048, 1024, 1024), id, st > 0);
        }
        mma_commit(&bar[0]);
        mma_issued++;
    }
    if (ok) ok = wait_mma();
    if (ok) ok = consensus(mbar_wait(&bar[2], 0, abort_flag));  // k, v (and W, U~, q) have landed
    // ---------------- epilogue 3: dB_k^T, dB_v^T tiles; dv; dbeta / dg partial sums ----------------
    if (ok) {
        float x[32], y[32];
        const int c = lr;  // key channel for dB_k^T, value channel for dB_v^T
        tmem_row32(tl + TM_DBK, x);
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) st_chunk(sm + R_S, swz(c, hf * 4 + c4), x + c4 * 8);
        // e^{g_i} k_ic dB_k^T[c][i]  (-> dbeta, and beta_i times it -> dg)
#pragma unroll
        for (int t = 0; t < 32; ++t) y[t] = eg[col0 + t] * ld_tile(sm + R_DO, col0 + t, c) * x[t];
        red_at(RK_KBK, quarter, col0 + lane) = warp_colsum32(y, lane);
        tmem_row32(tl + TM_DUT, x);
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) st_chunk(sm + R_S + 16384, swz(c, hf * 4 + c4), x + c4 * 8);
#pragma unroll
        for (int t = 0; t < 32; ++t) {
            const int i = col0 + t;
            y[t] = ld_tile(sm + R_KB, i, c) * x[t];
            st_tile(sm + R_DUT, i, c, betas[i] * x[t]);  // dv [i][j]
        }
        red_at(RK_VBV, quarter, col0 + lane) = warp_colsum32(y, lane);
    }
    fence_proxy_async();
    fence_before_sync();
    ok = consensus(ok);
    // ---------------- dv out; batch 4: dA' = dB_k W^T + dB_v U~^T  (rows 0..63 valid) ----------------
    if (ok && tid == 0) {
        fence_after_sync();
        tma_store_4d(&mp.dv, sm + R_DUT, 0, h, t0, b);
        tma_store_4d(&mp.dv, sm + R_DUT + 8192, 64, h, t0, b);
        bulk_commit();
        const uint32_t id = idesc_bf16(128, 64, 1, 0);
        const uint32_t sBk = sS, sBv = sS + 16384, sW = sD, sUt = sD + 16384;
#pragma unroll
        for (int st = 0; st < 16; ++st) {
            const uint32_t aa = (st < 8 ? sBk : sBv) + (st & 7) * 2048;
            const uint32_t bb = (st < 8 ? sW : sUt) + ((st & 7) >> 2) * 8192 + (st & 3) * 32;
            mma_bf16(tbase + TM_DW, sdesc(aa, 16384, 1024), sdesc(bb, 16, 1024), id, st > 0);
        }
        mma_commit(&bar[0]);
        mma_issued++;
    }
    if (ok) ok = wait_mma();
    // ---------------- epilogue 4 (rows r < 64): D_P, D_M, Z, dbeta (A part) ----------------
    if (ok && quarter < 2) {
        const int r = lr;
        float da[32], dp[32], pv[32], kk[32];
        tmem_row32(tl + TM_DW, da);
        tmem_row32(tl + TM_DP, dp);
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
            ld_chunk(sm + R_P, swz(r, hf * 4 + c4), pv + c4 * 8);
            ld_chunk(sm + R_KK, swz(r, hf * 4 + c4), kk + c4 * 8);
        }
        const float br = betas[r], gr = gc[r];
        float rowz = 0.f, dbA = 0.f;
#pragma unroll
        for (int t = 0; t < 32; ++t) {
            const int i = col0 + t;
            const float e = (i <= r) ? (gated ? __expf(gr - gc[i]) : 1.f) : 0.f;
            const float d = (i < r) ? -da[t] : 0.f;
            const float p = (i <= r) ? dp[t] : 0.f;
            const float dak = d * kk[t] * e;
            dbA += dak;
            const float z = p * pv[t] + br * dak;
            rowz += z;
            dp[t] = p * e;        // D_P
            da[t] = br * d * e;   // D_M
            pv[t] = z;
        }
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
            st_chunk(sm + R_P, swz(r, hf * 4 + c4), dp + c4 * 8);
            st_chunk(sm + R_T, swz(r, hf * 4 + c4), da + c4 * 8);
        }
        rowsum[hf * 64 + r] = rowz;
        rowsum[128 + hf * 64 + r] = dbA;
        red_at(RK_ZC, quarter, col0 + lane) = warp_colsum32(pv, lane);
    }
    fence_proxy_async();
    fence_before_sync();
    ok = consensus(ok);
    // ---------------- batch 5: dq^T = k^T D_P^T;  dk^T = q^T D_P + k^T D_M + k^T D_M^T ----------------
    if (ok && tid == 0) {
        fence_after_sync();
        const uint32_t sQ = sU, sKr = sO, sDP = sP, sDM = sT;
        const uint32_t id_q = idesc_bf16(128, 64, 1, 0), id_k = idesc_bf16(128, 64, 1, 1);
#pragma unroll
        for (int st = 0; st < 4; ++st) {
            mma_bf16(tbase + TM_DQ, sdesc(sKr + st * 2048, 8192, 1024), sdesc(sDP + st * 32, 16, 1024), id_q, st > 0);
            mma_bf16(tbase + TM_DK, sdesc(sQ + st * 2048, 8192, 1024), sdesc(sDP + st * 2048, 1024, 1024), id_k,
                     st > 0);
        }
#pragma unroll
        for (int st = 0; st < 4; ++st) {
            mma_bf16(tbase + TM_DK, sdesc(sKr + st * 2048, 8192, 1024), sdesc(sDM + st * 2048, 1024, 1024), id_k, 1);
            mma_bf16(tbase + TM_DK, sdesc(sKr + st * 2048, 8192, 1024), sdesc(sDM + st * 32, 16, 1024), id_q, 1);
        }
        mma_commit(&bar[0]);
        mma_issued++;
    }
    if (ok) ok = wait_mma();
    // ---------------- epilogue 5: dq, dk staging; dg channel sums ----------------
    if (ok) {
        const int c = lr;
        float w[32], acc[32], y[32];
        // dq = e^g (dO S^T) + D_P k ; dg += e^g q . (dO S^T)
        tmem_row32(tl + TM_QD, w);
        tmem_row32(tl + TM_DQ, acc);
#pragma unroll
        for (int t = 0; t < 32; ++t) {
            const int r = col0 + t;
            st_tile(sm + R_DWT, r, c, eg[r] * w[t] + acc[t]);
            y[t] = eg[r] * ld_tile(sm + R_U, r, c) * w[t];
        }
        red_at(RK_QQD, quarter, col0 + lane) = warp_colsum32(y, lane);
        // dk = D_P^T q + (D_M + D_M^T) k + beta e^g dB_k + e^{gC-g} U dS+^T ; dg terms
        float tm[32];
        tmem_row32(tl + TM_DK, acc);
        tmem_row32(tl + TM_DBK, w);
        tmem_row32(tl + TM_TM, tm);
#pragma unroll
        for (int t = 0; t < 32; ++t) {
            const int r = col0 + t;
            st_tile(sm + R_DS, r, c, acc[t] + betas[r] * eg[r] * w[t] + egc[r] * tm[t]);
            y[t] = egc[r] * ld_tile(sm + R_DO, r, c) * tm[t];
        }
        red_at(RK_KTM, quarter, col0 + lane) = warp_colsum32(y, lane);
    }
    fence_proxy_async();
    fence_before_sync();
    ok = consensus(ok);
    if (ok && tid == 0) {
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            tma_store_4d(&mp.dq, sm + R_DWT + p * 8192, 64 * p, h, t0, b);
            tma_store_4d(&mp.dk, sm + R_DS + p * 8192, 64 * p, h, t0, b);
        }
        bulk_commit();
    }
    // ---------------- dbeta, dg, d log alpha ----------------
    if (ok && tid < C) {
        const int r = tid;
        float sq = 0.f, sbk = 0.f, skt = 0.f, sv = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            sq += red_at(RK_QQD, q, r);
            sbk += red_at(RK_KBK, q, r);
            skt += red_at(RK_KTM, q, r);
            sv += red_at(RK_VBV, q, r);
        }
        const float zc = red_at(RK_ZC, 0, r) + red_at(RK_ZC, 1, r);
        const float rowz = rowsum[r] + rowsum[64 + r], dbA = rowsum[128 + r] + rowsum[192 + r];
        if (r < L) st_bf(a.dbeta, trow_g(r), dbA + sbk + sv);
        dgs[r] = rowz - zc + sq + betas[r] * sbk - skt;
        ktm[r] = skt;
    }
    __syncthreads();
    if (ok && gated && warp == 0) {
        float a0 = dgs[2 * lane], a1 = dgs[2 * lane + 1];
        const float tsum = warp_sum(ktm[2 * lane] + ktm[2 * lane + 1]);
        float rs = 0.f;
#pragma unroll
        for (int w8 = 0; w8 < 8; ++w8) rs += rsp[w8];
        // the chunk-end terms belong to dg_C (last row): the k . Tm sums and the decay
        // e^{g_C} of the incoming state
        if (lane == 31) a1 += tsum + __expf(gc[C - 1]) * rs;
        const float tot = a0 + a1;
        float incl = tot;  // inclusive suffix sum over lanes
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_down_sync(0xffffffffu, incl, o);
            if (lane + o < 32) incl += y;
        }
        const float excl = incl - tot;
        if (2 * lane < L) st_bf(a.dalpha, trow_g(2 * lane), tot + excl);
        if (2 * lane + 1 < L) st_bf(a.dalpha, trow_g(2 * lane + 1), a1 + excl);
    }
    if (tid == 0) {
        bulk_wait_all();
        if (*abort_flag) {  // let whatever was issued finish before the CTA leaves
            volatile int dummy = 0;
            if (mma_issued > 0) mbar_wait(&bar[0], (mma_issued - 1) & 1, &dummy, 100000000ull);
            if (loads_issued >= 1) mbar_wait(&bar[1], 0, &dummy, 100000000ull);
            if (loads_issued >= 2) mbar_wait(&bar[2], 0, &dummy, 100000000ull);
        }
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == 0) tmem_dealloc(tbase, TM_COLS);
}

}  // namespace tcb

cudaError_t tc_bwd_chunk(const Geo &g, const Tensors &t, const TcWs &w, cudaStream_t s, Rec &rec) {
    using namespace tcb;
    Maps mp;
    const uint64_t Bn = g.B, T = g.T, H = g.H, NC = (uint64_t)g.B * g.H * g.N;
    bool ok = tc::make_map_4d_bf16(&mp.q, t.q, DK, H, T, Bn, 64) && tc::make_map_4d_bf16(&mp.k, t.k, DK, H, T, Bn, 64) &&
              tc::make_map_4d_bf16(&mp.v, t.v, DV, H, T, Bn, 64) &&
              tc::make_map_4d_bf16(&mp.dout, t.dout, DV, H, T, Bn, 64) &&
              tc::make_map_4d_bf16(&mp.dq, t.dq, DK, H, T, Bn, 64) &&
              tc::make_map_4d_bf16(&mp.dk, t.dk, DK, H, T, Bn, 64) &&
              tc::make_map_4d_bf16(&mp.dv, t.dv, DV, H, T, Bn, 64) &&
              tc::make_map_2d_bf16(&mp.S, w.Sn, DV, NC * DK, 128) &&
              tc::make_map_2d_bf16(&mp.dS, w.dSn, DV, NC * DK, 128) &&
              tc::make_map_2d_bf16(&mp.U, w.Un, DV, NC * C, 64) && tc::make_map_2d_bf16(&mp.W, w.W, DK, NC * C, 64) &&
              tc::make_map_2d_bf16(&mp.Ut, w.Ut, DV, NC * C, 64) && tc::make_map_2d_bf16(&mp.P, w.P, C, NC * C, 64) &&
              tc::make_map_2d_bf16(&mp.T, w.Tn, C, NC * C, 64) && tc::make_map_2d_bf16(&mp.KK, w.KK, C, NC * C, 64);
    if (ok && t.du) ok = tc::make_map_4d_bf16(&mp.du, t.du, DV, H, T, Bn, 64);
    else mp.du = mp.dout;
    if (!ok) return cudaErrorInvalidValue;
    Args a;
    a.beta = t.beta; a.dalpha = t.dalpha; a.dbeta = t.dbeta; a.g = w.g;
    a.B = g.B; a.T = g.T; a.H = g.H; a.N = g.N; a.variant = g.variant; a.has_du = t.du != nullptr;
    const size_t smem = SMEM_BYTES + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_bwd_chunk_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    rec.mark(s);
    k_bwd_chunk_tc<<<dim3(g.N, g.H, g.B), NTHREADS, smem, s>>>(mp, a);
    return cudaGetLastError();
}

}  // namespace dr
