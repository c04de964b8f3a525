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
// shared memory and are discarded.  One CTA of 128 threads per chunk; thread t owns TMEM
// lane t.
#include "simt_path.cuh"
#include "tc_path.cuh"
#include "tc_ptx.cuh"
#include "tc_tile.cuh"

namespace dr {
namespace tcb {

using namespace dr::tc;
using dr::tcf::st_chunk;
using dr::tcf::tmem_row64;

constexpr int C = 64, DK = 128, DV = 128;
constexpr int NTHREADS = 128;
// shared memory (bytes from a 1024-aligned base); later phases reuse earlier regions
constexpr uint32_t R_S = 0;           // 32K  S [c][j]           -> dB_k^T [c][i] (16K) | dB_v^T [j][i] (16K)
constexpr uint32_t R_DS = 32768;      // 32K  dS+ [c][j]         -> W [i][c] (16K) | U~ [i][j] (16K)
constexpr uint32_t R_U = 65536;       // 16K  U [r][j]           -> q [r][c]
constexpr uint32_t R_DO = 81920;      // 16K  dO [r][j]          -> k [r][c]
constexpr uint32_t R_KB = 98304;      // 16K  Kbar [r][c]
constexpr uint32_t R_P = 114688;      //  8K  P [r'][r] (row-major) -> D_P [r][i]
constexpr uint32_t R_T = 122880;      //  8K  T [r][i]           -> D_M + D_M^T [r][i]
constexpr uint32_t R_DUT = 131072;    // 16K  dU^T [j][r]
constexpr uint32_t R_DWT = 147456;    // 16K  dW^T [c][r]
constexpr uint32_t R_F = 163840;      // 49K  fp32 64 x 65 scratch x 3: Pf, dPf, Zf
constexpr uint32_t R_MISC = R_F + 50176;
constexpr uint32_t SMEM_BYTES = R_MISC + 8192;
// misc (floats unless noted)
constexpr uint32_t M_BAR = 0, M_TMEM = 64, M_ABORT = 68;
constexpr uint32_t M_GC = 256, M_BETA = 512, M_EG = 768, M_EGC = 1024;   // [64] each
constexpr uint32_t M_RED = 1280;     // [3 kinds][4 warps][64]: q.Qd, k.dBk, k.Tm partial sums
constexpr uint32_t M_RDB = M_RED + 3 * 4 * 64 * 4;  // [2][4][64]: v.dBv, k.dBk (for dbeta)
constexpr uint32_t M_RS = M_RDB + 2 * 4 * 64 * 4;   // [4]: partial sums of S .* dS+
constexpr uint32_t M_DG = M_RS + 64;                // [64] dg
static_assert(M_DG + 256 <= 8192, "misc overflow");
static_assert(3 * 64 * 65 * 4 <= 50176, "fp32 scratch overflow");
// TMEM columns
constexpr uint32_t TM_DUT = 0, TM_QD = 64, TM_TM = 128, TM_DP = 192, TM_DW = 256, TM_DBK = 320, TM_DQ = 384,
                   TM_DK = 448, TM_COLS = 512;
// fp32 scratch (row stride 65 floats)
constexpr int LD = 65;

struct Args {
    const void *q, *k, *v, *alpha, *beta, *dout, *du;  // bf16
    void *dq, *dk, *dv, *dalpha, *dbeta;                // bf16
    SimtWs w;
    int B, T, H, N, variant;
};

__device__ __forceinline__ void ld8f(const float *p, float *v) {
    const float4 a = reinterpret_cast<const float4 *>(p)[0], b = reinterpret_cast<const float4 *>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void ld8h(const void *p, float *v) {
    const uint4 w = *reinterpret_cast<const uint4 *>(p);
    v[0] = bf16_lo(w.x); v[1] = bf16_hi(w.x); v[2] = bf16_lo(w.y); v[3] = bf16_hi(w.y);
    v[4] = bf16_lo(w.z); v[5] = bf16_hi(w.z); v[6] = bf16_lo(w.w); v[7] = bf16_hi(w.w);
}

__device__ __forceinline__ float bfv(const void *p, size_t i) {
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i]);
}

__device__ __forceinline__ void st_bf(void *p, size_t i, float x) {
    reinterpret_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(x);
}

// sum over the 128 threads of per-thread values x[r] (r = 0..63), via warp shuffles and
// red[4][64]; the result for row r is available in red[0][r] + ... + red[3][r] after a sync.
__device__ __forceinline__ void warp_partial_rows(const float *x, float *red, int warp, int lane) {
#pragma unroll 4
    for (int r = 0; r < C; ++r) {
        float v = x[r];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[warp * C + r] = v;
    }
}

__global__ void __launch_bounds__(NTHREADS, 1) k_bwd_chunk_tc(Args a) {
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
    float *rdb = reinterpret_cast<float *>(sm + R_MISC + M_RDB);
    float *rsp = reinterpret_cast<float *>(sm + R_MISC + M_RS);
    float *dgs = reinterpret_cast<float *>(sm + R_MISC + M_DG);
    float *Pf = reinterpret_cast<float *>(sm + R_F);
    float *dPf = Pf + 64 * LD;
    float *Zf = dPf + 64 * LD;

    const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int T = a.T, H = a.H, t0 = n * C, L = min(C, T - t0);
    const size_t ci = ((size_t)b * H + h) * a.N + n;
    const bool gated = a.variant == VAR_GATED;
    auto trow_g = [&](int r) -> size_t { return ((size_t)b * T + t0 + r) * H + h; };  // token row (r < L)

    if (tid == 0) {
        mbar_init(bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, TM_COLS);

    // ---------------- phase 0: factors and bf16 operand tiles ----------------
    const float *Gg = a.w.G + ci * C * DK;
    if (tid < C) {
        const int r = tid;
        const float x = Gg[(size_t)r * DK];
        gc[r] = x;
        betas[r] = (r < L) ? bfv(a.beta, trow_g(r)) : 0.f;
        eg[r] = __expf(x);
        egc[r] = __expf(Gg[(size_t)(C - 1) * DK] - x);
    }
    if (tid < 4) rsp[tid] = 0.f;
    __syncthreads();
    const float *Sg = a.w.Sn + ci * DK * DV, *dSg = a.w.dSn + ci * DK * DV;
    float rs_part = 0.f;
    for (int x = tid; x < DK * 16; x += NTHREADS) {  // S, dS+ : 128 rows x 16 chunks of 8
        const int r = x >> 4, c16 = x & 15, p = c16 >> 3, ch = c16 & 7;
        float v[8], w[8];
        ld8f(Sg + (size_t)r * DV + c16 * 8, v);
        ld8f(dSg + (size_t)r * DV + c16 * 8, w);
#pragma unroll
        for (int e = 0; e < 8; ++e) rs_part += v[e] * w[e];
        st_chunk(sm + R_S, (uint32_t)p * 16384 + swz(r, ch), v);
        st_chunk(sm + R_DS, (uint32_t)p * 16384 + swz(r, ch), w);
    }
    const float *Ug = a.w.Un + ci * C * DV;
    for (int x = tid; x < C * 16; x += NTHREADS) {  // U, dO, Kbar : 64 rows x 16 chunks
        const int r = x >> 4, c16 = x & 15, p = c16 >> 3, ch = c16 & 7;
        const uint32_t o = (uint32_t)p * 8192 + swz(r, ch);
        float v[8];
        ld8f(Ug + (size_t)r * DV + c16 * 8, v);
        st_chunk(sm + R_U, o, v);
        if (r < L) ld8h(reinterpret_cast<const __nv_bfloat16 *>(a.dout) + trow_g(r) * DV + c16 * 8, v);
        else
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = 0.f;
        st_chunk(sm + R_DO, o, v);
        if (r < L) {
            ld8h(reinterpret_cast<const __nv_bfloat16 *>(a.k) + trow_g(r) * DK + c16 * 8, v);
            const float f = egc[r];
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] *= f;
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = 0.f;
        }
        st_chunk(sm + R_KB, o, v);
    }
    const float *Pg = a.w.P + ci * C * C, *Tg = a.w.Tn + ci * C * C;
    for (int x = tid; x < C * 8; x += NTHREADS) {  // P, T : 64 rows x 8 chunks
        const int r = x >> 3, ch = x & 7;
        float v[8];
        ld8f(Pg + (size_t)r * C + ch * 8, v);
        st_chunk(sm + R_P, swz(r, ch), v);
#pragma unroll
        for (int e = 0; e < 8; ++e) Pf[r * LD + ch * 8 + e] = v[e];
        ld8f(Tg + (size_t)r * C + ch * 8, v);
        st_chunk(sm + R_T, swz(r, ch), v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) rs_part += __shfl_xor_sync(0xffffffffu, rs_part, o);
    if (lane == 0) rsp[warp] = rs_part;
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tl = tbase + ((uint32_t)(warp * 32) << 16);
    uint32_t phase = 0;
    bool ok = true;
    auto mma_round = [&]() {
        mma_commit(bar);
        return;
    };
    auto wait_mma = [&]() -> bool {
        mbar_wait(bar, phase & 1, abort_flag);
        phase++;
        fence_after_sync();
        return !named_sync_any(1, NTHREADS, *abort_flag != 0);
    };
    const uint32_t sS = smem_u32(sm + R_S), sD = smem_u32(sm + R_DS), sU = smem_u32(sm + R_U);
    const uint32_t sO = smem_u32(sm + R_DO), sK = smem_u32(sm + R_KB), sP = smem_u32(sm + R_P);
    const uint32_t sT = smem_u32(sm + R_T), sUT = smem_u32(sm + R_DUT), sWT = smem_u32(sm + R_DWT);

    // ---------------- batch 1: dU^T, Qd^T, Tm^T, dP ----------------
    if (tid == 0) {
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
        mma_round();
    }
    ok = wait_mma();
    // ---------------- epilogue 1: dU (-> dU^T tile), dP rows ----------------
    if (ok) {
        float v[64];
        tmem_row64(tl + TM_DUT, v);
        const int j = tid;
        if (a.du)
            for (int r = 0; r < L; ++r) v[r] += bfv(a.du, trow_g(r) * DV + j);
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) st_chunk(sm + R_DUT, swz(j, ch), v + ch * 8);
        if (tid < C) {
            const int r = tid;
            tmem_row64(tl + TM_DP, v);
#pragma unroll
            for (int i = 0; i < 64; ++i) dPf[r * LD + i] = (i <= r) ? v[i] : 0.f;
        }
    }
    fence_proxy_async();
    fence_before_sync();
    ok = ok && !named_sync_any(1, NTHREADS, *abort_flag != 0);
    // ---------------- batch 2: dW^T = -S dU^T ----------------
    if (ok && tid == 0) {
        fence_after_sync();
        const uint32_t id = idesc_bf16(128, 64, 0, 1, 1);
#pragma unroll
        for (int st = 0; st < 8; ++st)
            mma_bf16(tbase + TM_DW, sdesc(sS + (st >> 2) * 16384 + (st & 3) * 32, 16, 1024),
                     sdesc(sUT + st * 2048, 1024, 1024), id, st > 0);
        mma_round();
    }
    if (ok) ok = wait_mma();
    if (ok) {
        float v[64];
        tmem_row64(tl + TM_DW, v);
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) st_chunk(sm + R_DWT, swz(tid, ch), v + ch * 8);
    }
    fence_proxy_async();
    fence_before_sync();
    ok = ok && !named_sync_any(1, NTHREADS, *abort_flag != 0);
    // ---------------- batch 3: dB_k^T = dW^T T, dB_v^T = dU^T T ----------------
    if (ok && tid == 0) {
        fence_after_sync();
        const uint32_t id = idesc_bf16(128, 64, 0, 1);
#pragma unroll
        for (int st = 0; st < 4; ++st) {
            mma_bf16(tbase + TM_DBK, sdesc(sWT + st * 32, 16, 1024), sdesc(sT + st * 2048, 1024, 1024), id, st > 0);
            mma_bf16(tbase + TM_DUT, sdesc(sUT + st * 32, 16, 1024), sdesc(sT + st * 2048, 1024, 1024), id, st > 0);
        }
        mma_round();
    }
    if (ok) ok = wait_mma();
    // ---------------- epilogue 3: tiles dB_k^T, dB_v^T; dv; dbeta / dg partial sums ----------------
    if (ok) {
        float x[64], y[64];
        const int c = tid;  // key channel for dB_k^T, value channel for dB_v^T
        tmem_row64(tl + TM_DBK, x);
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) st_chunk(sm + R_S, swz(c, ch), x + ch * 8);
        // e^{g_i} k_ic dB_k^T[c][i]  (-> dbeta, and beta_i times it -> dg)
        for (int i = 0; i < C; ++i) y[i] = (i < L) ? eg[i] * bfv(a.k, trow_g(i) * DK + c) * x[i] : 0.f;
        warp_partial_rows(y, rdb + 4 * C, warp, lane);
        tmem_row64(tl + TM_DUT, x);
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) st_chunk(sm + R_S + 16384, swz(c, ch), x + ch * 8);
        for (int i = 0; i < C; ++i) {
            float vv = 0.f;
            if (i < L) {
                vv = bfv(a.v, trow_g(i) * DV + c);
                st_bf(a.dv, trow_g(i) * DV + c, betas[i] * x[i]);
            }
            y[i] = vv * x[i];
        }
        warp_partial_rows(y, rdb, warp, lane);
    }
    // W, U~ -> tiles (dS+ no longer needed)
    {
        const float *Wg = a.w.W + ci * C * DK, *Utg = a.w.Ut + ci * C * DV;
        for (int x = tid; x < C * 16; x += NTHREADS) {
            const int r = x >> 4, c16 = x & 15, p = c16 >> 3, ch = c16 & 7;
            float v[8];
            ld8f(Wg + (size_t)r * DK + c16 * 8, v);
            st_chunk(sm + R_DS, (uint32_t)p * 8192 + swz(r, ch), v);
            ld8f(Utg + (size_t)r * DV + c16 * 8, v);
            st_chunk(sm + R_DS + 16384, (uint32_t)p * 8192 + swz(r, ch), v);
        }
    }
    fence_proxy_async();
    fence_before_sync();
    ok = ok && !named_sync_any(1, NTHREADS, *abort_flag != 0);
    // ---------------- batch 4: dA' = dB_k W^T + dB_v U~^T  (rows 0..63 valid) ----------------
    if (ok && tid == 0) {
        fence_after_sync();
        const uint32_t id = idesc_bf16(128, 64, 1, 0);
        const uint32_t sBk = sS, sBv = sS + 16384, sW = sD, sUt = sD + 16384;
#pragma unroll
        for (int st = 0; st < 16; ++st) {
            const uint32_t aa = (st < 8 ? sBk : sBv) + (st & 7) * 2048;
            const uint32_t bb = (st < 8 ? sW : sUt) + ((st & 7) >> 2) * 8192 + (st & 3) * 32;
            mma_bf16(tbase + TM_DW, sdesc(aa, 16384, 1024), sdesc(bb, 16, 1024), id, st > 0);
        }
        mma_round();
    }
    if (ok) ok = wait_mma();
    // ---------------- epilogue 4: D_P, D_M, Z, dbeta (A part) ----------------
    float dbA = 0.f;
    if (ok && tid < C) {
        const int r = tid;
        float v[64];
        tmem_row64(tl + TM_DW, v);
        const float *KKg = a.w.KK + ci * C * C + (size_t)r * C;
        const float br = betas[r], grr = gc[r];
        float rowz = 0.f;
        float dp[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            const float e = gated ? __expf(grr - gc[i]) : 1.f;
            const float da = (i < r) ? -v[i] : 0.f;
            const float kk = KKg[i];
            dbA += da * kk * e;
            const float dpi = dPf[r * LD + i];
            const float z = dpi * Pf[r * LD + i] + da * br * kk * e;
            rowz += z;
            Zf[r * LD + i] = z;
            dp[i] = dpi * e;                 // D_P row r
            v[i] = br * da * e;              // D_M row r
        }
        dgs[r] = rowz;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) st_chunk(sm + R_P, swz(r, ch), dp + ch * 8);
#pragma unroll
        for (int i = 0; i < 64; ++i) dPf[r * LD + i] = v[i];  // D_M (dP no longer needed)
    }
    __syncthreads();
    if (ok && tid < C) {
        const int r = tid;
        float sym[64], colz = 0.f;
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            sym[i] = dPf[r * LD + i] + dPf[i * LD + r];
            colz += Zf[i * LD + r];
        }
        dgs[r] -= colz;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) st_chunk(sm + R_T, swz(r, ch), sym + ch * 8);
    }
    // q, k -> tiles (U, dO no longer needed)
    for (int x = tid; x < C * 16; x += NTHREADS) {
        const int r = x >> 4, c16 = x & 15, p = c16 >> 3, ch = c16 & 7;
        const uint32_t o = (uint32_t)p * 8192 + swz(r, ch);
        float v[8];
        if (r < L) ld8h(reinterpret_cast<const __nv_bfloat16 *>(a.q) + trow_g(r) * DK + c16 * 8, v);
        else
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = 0.f;
        st_chunk(sm + R_U, o, v);
        if (r < L) ld8h(reinterpret_cast<const __nv_bfloat16 *>(a.k) + trow_g(r) * DK + c16 * 8, v);
        else
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = 0.f;
        st_chunk(sm + R_DO, o, v);
    }
    fence_proxy_async();
    fence_before_sync();
    ok = ok && !named_sync_any(1, NTHREADS, *abort_flag != 0);
    // ---------------- batch 5: dq^T += k^T D_P^T;  dk^T = q^T D_P + k^T (D_M + D_M^T) ----------------
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
        for (int st = 0; st < 4; ++st)
            mma_bf16(tbase + TM_DK, sdesc(sKr + st * 2048, 8192, 1024), sdesc(sDM + st * 2048, 1024, 1024), id_k, 1);
        mma_round();
    }
    if (ok) ok = wait_mma();
    // ---------------- epilogue 5: dq, dk; dg channel sums ----------------
    if (ok) {
        const int c = tid;
        float acc[64], w[64], x[64];
        // dq = e^g (dO S^T) + D_P k ; dg += e^g q . (dO S^T)
        tmem_row64(tl + TM_QD, w);
        tmem_row64(tl + TM_DQ, acc);
        for (int r = 0; r < C; ++r) {
            float qv = 0.f;
            if (r < L) {
                qv = bfv(a.q, trow_g(r) * DK + c);
                st_bf(a.dq, trow_g(r) * DK + c, eg[r] * w[r] + acc[r]);
            }
            x[r] = eg[r] * qv * w[r];
        }
        warp_partial_rows(x, red, warp, lane);
        // dk = D_P^T q + (D_M + D_M^T) k + beta e^g dB_k + e^{gC-g} U dS+^T ; dg terms
        tmem_row64(tl + TM_DK, acc);
        tmem_row64(tl + TM_DBK, w);
        float y[64];
        tmem_row64(tl + TM_TM, y);
        float tsum = 0.f;
        for (int r = 0; r < C; ++r) {
            float kv = 0.f;
            if (r < L) {
                kv = bfv(a.k, trow_g(r) * DK + c);
                st_bf(a.dk, trow_g(r) * DK + c, acc[r] + betas[r] * eg[r] * w[r] + egc[r] * y[r]);
            }
            x[r] = egc[r] * kv * y[r];
            tsum += x[r];
        }
        warp_partial_rows(x, red + 2 * 4 * C, warp, lane);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) tsum += __shfl_xor_sync(0xffffffffu, tsum, o);
        // the chunk-end term sum_r e^{g_C - g_r} k_r . (U dS+^T)_r belongs to dg_C (last row)
        if (lane == 0) atomicAdd(&dgs[C - 1], tsum);
    }
    __syncthreads();
    // ---------------- dbeta, dg, d log alpha ----------------
    if (ok && tid < C) {
        const int r = tid;
        float sq = 0.f, sbk = 0.f, skt = 0.f, sv = 0.f;
#pragma unroll
        for (int w4 = 0; w4 < 4; ++w4) {
            sq += red[w4 * C + r];
            skt += red[2 * 4 * C + w4 * C + r];
            sv += rdb[w4 * C + r];
            sbk += rdb[4 * C + w4 * C + r];
        }
        if (r < L) st_bf(a.dbeta, trow_g(r), dbA + sbk + sv);
        dgs[r] += sq + betas[r] * sbk - skt;
    }
    __syncthreads();
    if (ok && gated && tid == 0) {
        float rs = 0.f;
#pragma unroll
        for (int w4 = 0; w4 < 4; ++w4) rs += rsp[w4];
        float run = __expf(gc[C - 1]) * rs;  // the chunk-end decay e^{g_C} of the incoming state
        for (int r = C - 1; r >= 0; --r) {
            run += dgs[r];
            if (r < L) st_bf(a.dalpha, trow_g(r), run);
        }
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == 0) tmem_dealloc(tbase, TM_COLS);
}

}  // namespace tcb

cudaError_t tc_bwd_chunk(const Geo &g, const Tensors &t, const SimtWs &w, cudaStream_t s, Rec &rec) {
    using namespace tcb;
    Args a;
    a.q = t.q; a.k = t.k; a.v = t.v; a.alpha = t.alpha; a.beta = t.beta; a.dout = t.dout; a.du = t.du;
    a.dq = t.dq; a.dk = t.dk; a.dv = t.dv; a.dalpha = t.dalpha; a.dbeta = t.dbeta;
    a.w = w;
    a.B = g.B; a.T = g.T; a.H = g.H; a.N = g.N; a.variant = g.variant;
    const size_t smem = SMEM_BYTES + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_bwd_chunk_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    rec.mark(s);
    k_bwd_chunk_tc<<<dim3(g.N, g.H, g.B), NTHREADS, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace dr
