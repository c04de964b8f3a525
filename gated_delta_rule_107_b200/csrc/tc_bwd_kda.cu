// tc_bwd_kda.cu -- KDA's intra-chunk gradients on tcgen05 (bf16, dk = dv = 128, C = 64).
//
// Backward of the chunked form of "线性注意力架构演进与Kimi Delta Attention创新实践" (sections
// 2.1, 2.2, 6.2, 7.1) for one chunk of one (b, h), with channel-wise gates.  With g[r][c] the
// in-chunk cumulative log gate, S = S_n, dS+ = dL/dS_{n+1}, dU = dL/dU (the reverse chain's), U,
// W, U~, T = (I + A)^-1 and M[r][i] = sum_c k_rc k_ic e^{g_rc - g_ic} (the forward's, kept):
//   Qd = dO S^T,  dWm = -dU S^T,  Tm = U dS+^T,  RS_c = sum_j S_cj dS+_cj
//   dB_k = T^T dWm,  dB_v = T^T dU
//   dA = -strict_tril(dB_k W^T + dB_v U~^T),  dM = diag(beta) dA,  dP = tril(dO U^T)
//   X_rc  = sum_i dP_ri k_ic e^{g_rc - g_ic},   Yv_rc = sum_i dM_ri k_ic e^{g_rc - g_ic}
//   Z_ic  = sum_r (dM_ri k_rc + dP_ri q_rc) e^{g_rc - g_ic}
//   dq = e^g Qd + X,   dk = Yv + Z + beta e^g dB_k + e^{g_C - g} Tm,   dv = diag(beta) dB_v
//   dg = q dq + k (Yv - Z) + beta e^g k dB_k - k e^{g_C - g} Tm;  dg_C += sum_r k e^{g_C - g} Tm + e^{g_C} RS
//   dbeta_r = sum_i dA_ri M_ri + e^g k . dB_k + v . dB_v;   d log alpha = reverse cumsum of dg
//
// Every per-(token, channel) quantity is formed channel-major -- the transposed product, with the
// key channel c as the 128-row side -- so that TMEM lane c holds channel c of every token: the
// gate factors, the chunk-end terms and the reverse cumulative sum are then per-thread work, and
// each warp's stores cover 32 consecutive channels.  The pair factors e^{g_rc - g_ic} are split at
// a token of each 16-token block (as in the forward): for X and Yv at the first token b of row
// r's block (operand sections Km_R = k_i e^{g_b - g_i}), for Z at the last token e of row i's
// block (Kp_I = k_r e^{g_r - g_e}, Qp_I likewise); every factor outside the diagonal block is
// <= 1, inside it at most e^{the block's fall}.  Chunks whose gate falls more than KDA_DIAG_SPAN
// inside a block are left to the CUDA-core gradient kernel (this kernel skips them).
//
// One CTA of 256 threads per chunk (two threads per key channel: warps w and w + 4 share TMEM
// lane quarter w, and split each epilogue's token columns in halves), phases in order:
//   A  loads; [Qd^T | -dWm^T] = S [dO ; dU]^T, Tm^T = dS+ U^T;  RS, g (from log alpha), dWm^T tile
//   B  loads of M, W, U~, v;  dB_k^T = dWm^T T,  dB_v^T = dU^T T;  their bf16 tiles, dv, v . dB_v
//   C  dA' = dB [W | U~]^T, [dO ; U][dO ; U]^T (dP and dP^T in one product);
//      dM, dP, dM^T, dP^T tiles, the dbeta part of A;  the gate-scaled sections Km, Kp, Qp
//   D  X^T, Yv^T, Z^T (block by block, N = 16);  the final per-channel epilogue
// Sums over the channels of one token (dbeta's) reduce 4 tokens at a time across a warp's 32 lanes
// (6 shuffles), then over the four warps of a lane quarter through shared memory.  The per-token
// loops are rolled over groups of 4 or 8 tokens (TMEM loads of 4 or 8 columns), so that every
// phase runs from a small loop body instead of long straight-line code.
// Every wait is bounded (~1 s); an expired wait raises the device error word.
#include "tc_host.cuh"
#include "tc_path.cuh"
#include "tc_ptx.cuh"
#include "tc_tile.cuh"

namespace dr {
namespace tck {

using namespace dr::tc;
using dr::tcf::ld_chunk;
using dr::tcf::st_chunk;

constexpr int C = 64, DK = 128, DV = 128;
constexpr int NTHREADS = 256;
// shared memory (bytes from a 1024-aligned base); regions are reused phase by phase
//   phase A:   S [0, 32K), dS+ [32K, 64K), [dO ; dU] [64K, 96K), [dO ; U] [96K, 128K),
//              T [128K, 136K), log alpha [136K, 152K), q [152K, 168K), k [168K, 184K)
//   E0 writes: G (fp32) [184K, 216K), dWm^T [136K, 152K) (after log alpha is read)
//   phase B:   M [0, 8K), W [8K, 24K), U~ [24K, 40K), v [40K, 56K) (dS+ is read by then);
//              E1 writes dB_k^T [64K, 80K), dB_v^T [80K, 96K)
//   E2 writes: dM [120K, 128K), dP [128K, 136K), dM^T [136K, 144K), dP^T [144K, 152K)
//   build:     Km [0, 40K), Kp [40K, 80K), Qp [80K, 120K)
constexpr uint32_t R_S = 0, R_DS = 32768, R_OU = 65536, R_OV = 98304, R_T = 131072, R_AL = 139264;
constexpr uint32_t R_Q = 155648, R_K = 172032, R_G = 188416, R_DWM = 139264;
constexpr uint32_t R_M = 0, R_W = 8192, R_UT = 24576, R_V = 40960, R_DBK = 65536, R_DBV = 81920;
constexpr uint32_t R_DM = 122880, R_DP = 131072, R_DMT = 139264, R_DPT = 147456;
constexpr uint32_t R_KM = 0, R_KP = 40960, R_QP = 81920;
constexpr uint32_t SEC_PANEL = KDA_KH_ROWS * 128;  // 160 rows x 128 B: one 64-channel panel of a section set
constexpr uint32_t R_MISC = R_G + 32768;           // 216K
// misc: barriers, TMEM slot, abort flag, then per-token and per-channel vectors (floats)
constexpr uint32_t M_BAR = 0;  // [0] phase-A loads, [1] phase-B loads, [2] MMA
constexpr uint32_t M_TMEM = 32, M_ABORT = 36;
constexpr uint32_t M_BETA = 64;          // [64] beta
constexpr uint32_t M_DBA = M_BETA + 256;  // [64] the dbeta part of A
constexpr uint32_t M_RED = M_DBA + 256;   // [2 kinds][4 lane quarters][64 tokens] dbeta partial sums
constexpr uint32_t M_XCH = M_RED + 2048;  // [2 halves][3][128]: dg_C and RS partials, the upper half's dg sum
constexpr uint32_t SMEM_BYTES = R_MISC + M_XCH + 3 * 2 * 128 * 4;
static_assert(SMEM_BYTES <= 227 * 1024 - 1024, "shared memory");
static_assert(R_V + 16384 <= R_DS + 32768 && R_V >= R_UT + 16384, "v tile inside the dead dS+ tile");
// TMEM columns (lane = key channel c, or value channel j for dB_v^T, or token row for dA', dP)
constexpr uint32_t TM_QD = 0, TM_X = 64, TM_TM = 128, TM_DBK = 192, TM_DBV = 256, TM_YV = 320, TM_D5 = 384,
                   TM_Z = 384, TM_COLS = 512;
constexpr uint32_t LOADA_BYTES = 4 * 32768 + 8192 + 3 * 16384, LOADB_BYTES = 8192 + 3 * 16384;

struct Maps {
    CUtensorMap q, k, v, dout, alpha;  // [B, T, H, 128] bf16; box 64 channels x 64 tokens
    CUtensorMap S, dS;              // [chunks * 128][128] bf16; box 64 x 128
    CUtensorMap U, dU, W, Ut;       // [chunks * 64][128] bf16; box 64 x 64
    CUtensorMap T, M;               // [chunks * 64][64] bf16; box 64 x 64
};

struct Args {
    const __nv_bfloat16 *beta;  // [B, T, H]
    __nv_bfloat16 *dq, *dk, *dv, *dalpha, *dbeta;
    const int *kwide;               // [chunks]: left to the CUDA-core kernel
    int T, H, N;
    int m0, m1;                     // the chunks [m0, m1) of each sequence (m1 = 0: all)
};

// first row of Km's section R (rows i = 0 .. 16 R + 15) and of Kp's / Qp's section I (rows 16 I .. 63)
__host__ __device__ constexpr int km_sec(int R) { return 8 * R * (R + 1); }
__host__ __device__ constexpr int kp_sec(int I) { return 64 * I - 8 * I * (I - 1); }
static_assert(km_sec(4) == KDA_KH_ROWS && kp_sec(4) == KDA_KH_ROWS, "160 rows per section set");

// element (row, c) of a [rows][128] bf16 tile stored as two 64-column swizzled panels of `panel` bytes
__device__ __forceinline__ uint32_t el_off(int row, int c, uint32_t panel) {
    return (uint32_t)(c >> 6) * panel + swz(row, (c & 63) >> 3) + (c & 7) * 2;
}
__device__ __forceinline__ float ld_bf(const unsigned char *base, uint32_t off) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(base + off));
}
// x[t] (t < 4) summed over the warp's lanes: two halving steps, then a plain sum over the
// remaining lane bits; afterwards every lane l holds the sum of token l / 8
__device__ __forceinline__ float warp_sum4(float (&x)[4], int lane) {
    const bool u16 = (lane & 16) != 0, u8 = (lane & 8) != 0;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float send = u16 ? x[i] : x[i + 2], keep = u16 ? x[i + 2] : x[i];
        x[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
    float v = (u8 ? x[1] : x[0]) + __shfl_xor_sync(0xffffffffu, u8 ? x[0] : x[1], 8);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    return v;
}
// 8 consecutive floats of a [64][128] fp32 tile (c0 a multiple of 8).  The two 16-byte halves are
// read in an order that depends on bit 2 of c0 / 8, so that the eight threads of a quarter warp
// reading one row at c0 = 0, 8, ..., 56 (or 64, ..., 120) hit eight different 4-bank groups.
__device__ __forceinline__ void ld_g8(const float *G, int row, int c0, float *o) {
    const int h = (c0 >> 5) & 1;
    const float4 a = *reinterpret_cast<const float4 *>(G + row * 128 + c0 + 4 * h);
    const float4 b = *reinterpret_cast<const float4 *>(G + row * 128 + c0 + 4 * (1 - h));
    const float lo[4] = {h ? b.x : a.x, h ? b.y : a.y, h ? b.z : a.z, h ? b.w : a.w};
    const float hi[4] = {h ? a.x : b.x, h ? a.y : b.y, h ? a.z : b.z, h ? a.w : b.w};
    o[0] = lo[0]; o[1] = lo[1]; o[2] = lo[2]; o[3] = lo[3]; o[4] = hi[0]; o[5] = hi[1]; o[6] = hi[2]; o[7] = hi[3];
}

__global__ void __launch_bounds__(NTHREADS, 1) k_bwd_kda_tc(const __grid_constant__ Maps mp, Args a) {
    const int ns = (a.m1 > 0 ? a.m1 : a.N) - a.m0;  // one CTA per chunk of the range, sequence by sequence
    const int ci = (int)(blockIdx.x / (unsigned)ns) * a.N + a.m0 + (int)(blockIdx.x % (unsigned)ns);
    if (a.kwide[ci]) return;  // uniform: the CUDA-core kernel takes this chunk
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    unsigned char *misc = sm + R_MISC;
    uint64_t *bar = reinterpret_cast<uint64_t *>(misc + M_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + M_TMEM);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + M_ABORT);
    float *betas = reinterpret_cast<float *>(misc + M_BETA);
    float *dba = reinterpret_cast<float *>(misc + M_DBA);
    float *red = reinterpret_cast<float *>(misc + M_RED);
    float *xch = reinterpret_cast<float *>(misc + M_XCH);
    const float *G = reinterpret_cast<const float *>(sm + R_G);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q4 = warp & 3, hf = warp >> 2;  // lane quarter; half of the token columns
    const int n = ci % a.N, bh = ci / a.N, h = bh % a.H, b = bh / a.H;
    const int T = a.T, H = a.H, t0 = n * C, L = min(C, T - t0);
    auto trow_g = [&](int rr) -> size_t { return ((size_t)b * T + t0 + rr) * H + h; };

    int armed[3] = {0, 0, 0};
    if (tid == 0) {
        for (int i = 0; i < 3; ++i) mbar_init(&bar[i], 1);
        *abort_flag = 0;
        fence_mbar_init();
        mbar_arrive_tx(&bar[0], LOADA_BYTES);
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            tma_load_2d(sm + R_S + p * 16384, &mp.S, 64 * p, ci * DK, &bar[0]);
            tma_load_2d(sm + R_DS + p * 16384, &mp.dS, 64 * p, ci * DK, &bar[0]);
            tma_load_4d(sm + R_OU + p * 16384, &mp.dout, 64 * p, h, t0, b, &bar[0]);
            tma_load_2d(sm + R_OU + p * 16384 + 8192, &mp.dU, 64 * p, ci * C, &bar[0]);
            tma_load_4d(sm + R_OV + p * 16384, &mp.dout, 64 * p, h, t0, b, &bar[0]);
            tma_load_2d(sm + R_OV + p * 16384 + 8192, &mp.U, 64 * p, ci * C, &bar[0]);
            tma_load_4d(sm + R_AL + p * 8192, &mp.alpha, 64 * p, h, t0, b, &bar[0]);
            tma_load_4d(sm + R_Q + p * 8192, &mp.q, 64 * p, h, t0, b, &bar[0]);
            tma_load_4d(sm + R_K + p * 8192, &mp.k, 64 * p, h, t0, b, &bar[0]);
        }
        tma_load_2d(sm + R_T, &mp.T, 0, ci * C, &bar[0]);
        armed[0] = 1;
    }
    if (tid < C) betas[tid] = tid < L ? __bfloat162float(a.beta[trow_g(tid)]) : 0.f;
    if (warp == 0) tmem_alloc(tmem_slot, TM_COLS);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tl = tbase + ((uint32_t)(q4 * 32) << 16);  // this warp's lane quarter
    auto consensus = [&](bool ok) -> bool { return !named_sync_any(1, NTHREADS, !ok || *abort_flag != 0); };
    uint32_t ph = 0;
    auto wait_mma = [&](bool also_ok) -> bool {
        const bool ok = mbar_wait(&bar[2], ph & 1, abort_flag);
        ph++;
        fence_after_sync();
        return consensus(ok && also_ok);
    };
    auto commit = [&]() {
        mma_commit(&bar[2]);
        armed[2]++;
    };
    auto u32 = [&](uint32_t off) { return smem_u32(sm + off); };
    const int c = tid & (DK - 1);  // this thread's key channel (TMEM lane); also value channel j = c
    const int r0 = 32 * hf;         // first token of this thread's column half

    bool ok = consensus(mbar_wait(&bar[0], 0, abort_flag));
    // ======================= phase A products =======================
    if (ok && tid == 0) {
        const uint32_t id0 = idesc_bf16(128, 128, 0, 0), id1 = idesc_bf16(128, 64, 0, 0);
#pragma unroll 1
        for (int k = 0; k < 8; ++k) {  // K = dv in steps of 16
            const uint32_t ka = (k >> 2) * 16384 + (k & 3) * 32;
            mma_bf16(tbase + TM_QD, sdesc(u32(R_S) + ka, 16, 1024), sdesc(u32(R_OU) + ka, 16, 1024), id0, k > 0);
            mma_bf16(tbase + TM_TM, sdesc(u32(R_DS) + ka, 16, 1024), sdesc(u32(R_OV) + 8192 + ka, 16, 1024), id1,
                     k > 0);
        }
        commit();
    }
    // while they run: g of channel c at this half's tokens (prefix sum over the chunk; tokens past T
    // add 0), and this half's part of RS_c (the state tiles' panel hf)
    if (ok) {
        float run = 0.f;
        float *Gw = reinterpret_cast<float *>(sm + R_G);
        if (hf) {
#pragma unroll 8
            for (int r = 0; r < 32; ++r) run += ld_bf(sm + R_AL, el_off(r, c, 8192));
        }
#pragma unroll 8
        for (int r = r0; r < r0 + 32; ++r) {
            run += ld_bf(sm + R_AL, el_off(r, c, 8192));
            Gw[r * DK + c] = run;
        }
        float rs = 0.f;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
            float s8[8], d8[8];
            const uint32_t o = (uint32_t)hf * 16384 + swz(c, ch);
            ld_chunk(sm + R_S, o, s8);
            ld_chunk(sm + R_DS, o, d8);
#pragma unroll
            for (int e = 0; e < 8; ++e) rs += s8[e] * d8[e];
        }
        xch[(hf * 3 + 1) * 128 + c] = rs;
    }
    ok = consensus(ok);  // the log-alpha tile is read: dWm^T may take its space
    if (ok) ok = wait_mma(true);
    if (ok) {
        // -dWm^T row c (TMEM columns 64..127 of [Qd^T | dU S^T]), this half's 32 tokens, as the
        // bf16 A operand of dB_k^T
        float v[32];
        tmem_ld16(tl + TM_QD + 64 + r0, v);
        tmem_ld16(tl + TM_QD + 80 + r0, v + 16);
        wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = -v[j];
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) st_chunk(sm + R_DWM, swz(c, 4 * hf + ch), v + ch * 8);
    }
    fence_proxy_async();
    fence_before_sync();
    ok = consensus(ok);
    // ======================= phase B =======================
    if (ok && tid == 0) {
        fence_after_sync();
        mbar_arrive_tx(&bar[1], LOADB_BYTES);
        tma_load_2d(sm + R_M, &mp.M, 0, ci * C, &bar[1]);
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            tma_load_2d(sm + R_W + p * 8192, &mp.W, 64 * p, ci * C, &bar[1]);
            tma_load_2d(sm + R_UT + p * 8192, &mp.Ut, 64 * p, ci * C, &bar[1]);
            tma_load_4d(sm + R_V + p * 8192, &mp.v, 64 * p, h, t0, b, &bar[1]);
        }
        armed[1] = 1;
        // dB_k^T = dWm^T T (A K-major [c][r]; B = T [r][i] MN-major)
        // dB_v^T = dU^T T  (A = dU [r][j] MN-major: the two 64-column panels 16K apart in [dO ; dU])
        const uint32_t idk = idesc_bf16(128, 64, 0, 1), idv = idesc_bf16(128, 64, 1, 1);
#pragma unroll 1
        for (int k = 0; k < 4; ++k) {
            mma_bf16(tbase + TM_DBK, sdesc(u32(R_DWM) + k * 32, 16, 1024), sdesc(u32(R_T) + k * 2048, 8192, 1024), idk,
                     k > 0);
            mma_bf16(tbase + TM_DBV, sdesc(u32(R_OU) + 8192 + k * 2048, 16384, 1024),
                     sdesc(u32(R_T) + k * 2048, 8192, 1024), idv, k > 0);
        }
        commit();
    }
    if (ok) ok = wait_mma(mbar_wait(&bar[1], 0, abort_flag));  // the products; M, W, U~, v
    if (ok) {
        // the bf16 tiles dB_k^T [c][i] and dB_v^T [j][i] (this half's 32 tokens), dv, and v . dB_v,
        // eight tokens at a time
#pragma unroll 1
        for (int k8 = 0; k8 < 4; ++k8) {
            const int rr = r0 + 8 * k8;
            float bk[8], bv[8];
            tmem_ld8(tl + TM_DBK + rr, bk);
            tmem_ld8(tl + TM_DBV + rr, bv);
            wait_ld();
            st_chunk(sm + R_DBK, swz(c, rr >> 3), bk);
            st_chunk(sm + R_DBV, swz(c, rr >> 3), bv);
            float s0[4], s1[4];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int r = rr + e;
                const float sv = ld_bf(sm + R_V, el_off(r, c, 8192)) * bv[e];
                if (e < 4) s0[e] = sv;
                else s1[e - 4] = sv;
                if (r < L) a.dv[trow_g(r) * DV + c] = __float2bfloat16_rn(betas[r] * bv[e]);
            }
            const float t0s = warp_sum4(s0, lane), t1s = warp_sum4(s1, lane);
            if ((lane & 7) == 0) {
                red[(4 + q4) * 64 + rr + (lane >> 3)] = t0s;
                red[(4 + q4) * 64 + rr + 4 + (lane >> 3)] = t1s;
            }
        }
    }
    fence_proxy_async();
    fence_before_sync();
    ok = consensus(ok);
    // ======================= phase C products =======================
    if (ok && tid == 0) {
        fence_after_sync();
        // dA'[r][i] = dB_k[r] . W[i] + dB_v[r] . U~[i]: A = dB^T tiles read MN-major (rows 64-127 of
        // the M = 128 product are discarded), B = W, U~ K-major
        const uint32_t ida = idesc_bf16(128, 64, 1, 0), id5 = idesc_bf16(128, 128, 0, 0);
#pragma unroll 1
        for (int k = 0; k < 16; ++k) {
            const uint32_t at = (k < 8 ? u32(R_DBK) : u32(R_DBV)) + (k & 7) * 2048;
            const uint32_t bw = (k < 8 ? u32(R_W) : u32(R_UT)) + ((k & 7) >> 2) * 8192 + (k & 3) * 32;
            mma_bf16(tbase + TM_X, sdesc(at, 8192, 1024), sdesc(bw, 16, 1024), ida, k > 0);
        }
        // [dO ; U] [dO ; U]^T: dP = dO U^T at lanes 0-63 / columns 64-127, dP^T at lanes 64-127 / 0-63
#pragma unroll 1
        for (int k = 0; k < 8; ++k) {
            const uint32_t ka = (k >> 2) * 16384 + (k & 3) * 32;
            mma_bf16(tbase + TM_D5, sdesc(u32(R_OV) + ka, 16, 1024), sdesc(u32(R_OV) + ka, 16, 1024), id5, k > 0);
        }
        commit();
    }
    if (ok) ok = wait_mma(true);
    // ---- E2: the masked tiles dM, dP [r][i] and dM^T, dP^T [i][r]; the dbeta part of A ----
    //   lanes 0-63 (quarters 0, 1): half 0 takes dA' (-> dM and, element by element at the
    //   transposed place, dM^T, dbeta_A), half 1 takes dP;  lanes 64-127: each half takes 32
    //   columns of dP^T
    if (ok) {
        const int rl = (warp & 1) * 32 + lane;  // the product's row (r, or i for the transposes)
        if (q4 < 2) {
            if (hf == 0) {
                const int r = rl;  // dA'[r][i] -> dM[r][i] = -beta_r dA' (i < r), dbeta_A
                float db = 0.f;
                const float br = betas[r];
#pragma unroll 1
                for (int ch = 0; ch < 8; ++ch) {
                    float x8[8], m8[8], w8[8];
                    tmem_ld8(tl + TM_X + 8 * ch, x8);
                    wait_ld();
                    ld_chunk(sm + R_M, swz(r, ch), m8);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float d = ch * 8 + e < r ? -x8[e] : 0.f;
                        db += d * m8[e];
                        w8[e] = br * d;
                        // dM^T[i][r] = dM[r][i]: the same bf16 at row i, column r
                        *reinterpret_cast<__nv_bfloat16 *>(sm + R_DMT + swz(ch * 8 + e, r >> 3) + (r & 7) * 2) =
                            __float2bfloat16_rn(w8[e]);
                    }
                    st_chunk(sm + R_DM, swz(r, ch), w8);
                }
                dba[r] = db;
            } else {
                const int r = rl;  // dP[r][i] (i <= r)
#pragma unroll 1
                for (int ch = 0; ch < 8; ++ch) {
                    float x8[8];
                    tmem_ld8(tl + TM_D5 + 64 + 8 * ch, x8);
                    wait_ld();
#pragma unroll
                    for (int e = 0; e < 8; ++e) x8[e] = ch * 8 + e <= r ? x8[e] : 0.f;
                    st_chunk(sm + R_DP, swz(r, ch), x8);
                }
            }
        } else {
            const int i = rl;  // dP^T[i][r] (r >= i), r in this half
#pragma unroll 1
            for (int k8 = 0; k8 < 4; ++k8) {
                const int rr = r0 + 8 * k8;
                float x8[8];
                tmem_ld8(tl + TM_D5 + rr, x8);
                wait_ld();
#pragma unroll
                for (int e = 0; e < 8; ++e) x8[e] = rr + e >= i ? x8[e] : 0.f;
                st_chunk(sm + R_DPT, swz(i, rr >> 3), x8);
            }
        }
    }
    ok = consensus(ok);  // M, W, U~ and the dB tiles are read: the sections may take their space
    // ---- the gate-scaled sections (thread = 16-byte chunk of a row, 8 channels) ----
    //   Km_R[i] = k_i e^{g_16R - g_i} (i <= 16 R + 15);  Kp_I[r] = k_r e^{g_r - g_{16 I + 15}},
    //   Qp_I[r] = q_r e^{g_r - g_{16 I + 15}} (r >= 16 I); exponents clamped at 80 (they exceed 0
    //   only inside a block, by at most KDA_DIAG_SPAN here)
    if (ok) {
        for (int x = tid; x < KDA_KH_ROWS * 16; x += NTHREADS) {
            const int row = x >> 4, cc = x & 15, c0 = cc * 8;
            const uint32_t o = (uint32_t)(cc >> 3) * SEC_PANEL + swz(row, cc & 7);
            // Km row: section R, token i
            int R = 0;
            while (R < 3 && row >= km_sec(R + 1)) ++R;
            const int ti = row - km_sec(R);
            // Kp / Qp row: section I, token r
            int I = 0;
            while (I < 3 && row >= kp_sec(I + 1)) ++I;
            const int tr = 16 * I + (row - kp_sec(I));
            float ki[8], kr[8], qr[8], gb[8], gi[8], gr[8], ge[8];
            ld_chunk(sm + R_K, (uint32_t)(c0 >> 6) * 8192 + swz(ti, (c0 & 63) >> 3), ki);
            ld_chunk(sm + R_K, (uint32_t)(c0 >> 6) * 8192 + swz(tr, (c0 & 63) >> 3), kr);
            ld_chunk(sm + R_Q, (uint32_t)(c0 >> 6) * 8192 + swz(tr, (c0 & 63) >> 3), qr);
            ld_g8(G, 16 * R, c0, gb);
            ld_g8(G, ti, c0, gi);
            ld_g8(G, tr, c0, gr);
            ld_g8(G, 16 * I + 15, c0, ge);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                ki[e] *= __expf(fminf(gb[e] - gi[e], 80.f));
                const float f = __expf(fminf(gr[e] - ge[e], 80.f));
                kr[e] *= f;
                qr[e] *= f;
            }
            st_chunk(sm + R_KM, o, ki);
            st_chunk(sm + R_KP, o, kr);
            st_chunk(sm + R_QP, o, qr);
        }
    }
    fence_proxy_async();
    fence_before_sync();
    ok = consensus(ok);
    // ======================= phase D products: X^T, Yv^T, Z^T (N = 16 per block) =======================
    if (ok && tid == 0) {
        fence_after_sync();
        const uint32_t id = idesc_bf16(128, 16, 1, 0);
#pragma unroll 1
        for (int R = 0; R < 4; ++R) {
#pragma unroll 1
            for (int kk = 0; kk <= R; ++kk) {  // tokens i of the blocks up to R
                const uint64_t am = sdesc(u32(R_KM) + (uint32_t)(km_sec(R) + 16 * kk) * 128, SEC_PANEL, 1024);
                mma_bf16(tbase + TM_X + 16 * R, am, sdesc(u32(R_DP) + 2048 * R + kk * 32, 16, 1024), id, kk > 0);
                mma_bf16(tbase + TM_YV + 16 * R, am, sdesc(u32(R_DM) + 2048 * R + kk * 32, 16, 1024), id, kk > 0);
            }
        }
#pragma unroll 1
        for (int I = 0; I < 4; ++I) {
#pragma unroll 1
            for (int kk = I; kk < 4; ++kk) {  // tokens r of the blocks from I on
                const uint32_t ro = (uint32_t)(kp_sec(I) + 16 * (kk - I)) * 128;
                mma_bf16(tbase + TM_Z + 16 * I, sdesc(u32(R_KP) + ro, SEC_PANEL, 1024),
                         sdesc(u32(R_DMT) + 2048 * I + kk * 32, 16, 1024), id, kk > I);
                mma_bf16(tbase + TM_Z + 16 * I, sdesc(u32(R_QP) + ro, SEC_PANEL, 1024),
                         sdesc(u32(R_DPT) + 2048 * I + kk * 32, 16, 1024), id, 1);
            }
        }
        commit();
    }
    if (ok) ok = wait_mma(true);
    // ======================= final epilogue: thread (c, half): tokens r0 .. r0 + 31, four at a time
    const float gL = G[(C - 1) * DK + c];
    float *DG = reinterpret_cast<float *>(sm + R_KM);  // [64][128] dg (the sections are read by now)
    if (ok) {
        float dgc = 0.f, tot = 0.f;
#pragma unroll 1
        for (int g4 = 0; g4 < 8; ++g4) {
            const int rr = r0 + 4 * g4, rb = rr >> 4;
            float qd[4], tm[4], bk[4], xx[4], yv[4], zz[4];
            tmem_ld4(tl + TM_QD + rr, qd);
            tmem_ld4(tl + TM_TM + rr, tm);
            tmem_ld4(tl + TM_DBK + rr, bk);
            tmem_ld4(tl + TM_X + rr, xx);
            tmem_ld4(tl + TM_YV + rr, yv);
            tmem_ld4(tl + TM_Z + rr, zz);
            wait_ld();
            const float gb = G[16 * rb * DK + c], ge = G[(16 * rb + 15) * DK + c];
            float sbk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = rr + e;
                const float g = G[r * DK + c], br = betas[r];
                const float qv = ld_bf(sm + R_Q, el_off(r, c, 8192)), kv = ld_bf(sm + R_K, el_off(r, c, 8192));
                const float gam = __expf(g), eb = __expf(gL - g);
                const float fb = __expf(g - gb), fe = __expf(fminf(ge - g, 80.f));
                const float X = fb * xx[e], Yv = fb * yv[e], Z = fe * zz[e];
                const float dq = gam * qd[e] + X;
                const float t = eb * tm[e], sb = br * gam * bk[e];
                const float dk = Yv + Z + sb + t;
                const float dg = qv * dq + kv * (Yv - Z + sb - t);
                DG[r * DK + c] = dg;
                tot += dg;
                dgc += kv * t;
                sbk[e] = gam * kv * bk[e];
                if (r < L) {
                    const size_t o = trow_g(r) * DK + c;
                    a.dq[o] = __float2bfloat16_rn(dq);
                    a.dk[o] = __float2bfloat16_rn(dk);
                }
            }
            const float s4 = warp_sum4(sbk, lane);
            if ((lane & 7) == 0) red[q4 * 64 + rr + (lane >> 3)] = s4;
        }
        xch[(hf * 3 + 0) * 128 + c] = dgc;
        if (hf) xch[(1 * 3 + 2) * 128 + c] = tot;
    }
    ok = consensus(ok);
    if (ok) {
        // d log alpha: the chunk-end terms (dg_C and e^{g_C} RS) belong to the last row, then the
        // reverse cumulative sum; the lower half starts from the upper half's total
        float run = xch[0 * 128 + c] + xch[3 * 128 + c] + __expf(gL) * (xch[1 * 128 + c] + xch[4 * 128 + c]);
        if (!hf) run += xch[5 * 128 + c];
        const size_t rstep = (size_t)H * DK;  // one token further in [B, T, H, 128]
        __nv_bfloat16 *da = a.dalpha + trow_g(r0 + 31) * DK + c;
#pragma unroll 4
        for (int e = 31; e >= 0; --e, da -= rstep) {
            run += DG[(r0 + e) * DK + c];
            if (r0 + e < L) *da = __float2bfloat16_rn(run);
        }
        if (tid < L) {
            float s = dba[tid];
#pragma unroll
            for (int w = 0; w < 4; ++w) s += red[w * 64 + tid] + red[(4 + w) * 64 + tid];
            a.dbeta[trow_g(tid)] = __float2bfloat16_rn(s);
        }
    }
    if (tid == 0 && *abort_flag) {  // let whatever was issued land before the CTA leaves
        volatile int dummy = 0;
        for (int i = 0; i < 2; ++i)
            if (armed[i] > 0) mbar_wait(&bar[i], 0, &dummy, 100000000ull);
        // every MMA batch ends with a commit: wait for the phases not waited for yet, in order
        for (uint32_t p = ph; p < (uint32_t)armed[2]; ++p) mbar_wait(&bar[2], p & 1, &dummy, 100000000ull);
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == 0) tmem_dealloc(tbase, TM_COLS);
}

}  // namespace tck

cudaError_t tc_bwd_kda(const Geo &g, const Tensors &t, const TcWs &w, cudaStream_t s, Rec &rec) {
    using namespace tck;
    Maps mp;
    const uint64_t Bn = g.B, T = g.T, H = g.H, NC = (uint64_t)g.B * g.H * g.N;
    bool ok = tc::make_map_4d_bf16(&mp.q, t.q, DK, H, T, Bn, 64) && tc::make_map_4d_bf16(&mp.k, t.k, DK, H, T, Bn, 64) &&
              tc::make_map_4d_bf16(&mp.v, t.v, DV, H, T, Bn, 64) &&
              tc::make_map_4d_bf16(&mp.alpha, t.alpha, DK, H, T, Bn, 64) &&
              tc::make_map_2d_bf16(&mp.S, w.Sn, DV, NC * DK, 128) && tc::make_map_2d_bf16(&mp.dS, w.dSn, DV, NC * DK, 128) &&
              tc::make_map_2d_bf16(&mp.U, w.Un, DV, NC * C, 64) && tc::make_map_2d_bf16(&mp.dU, w.dUn, DV, NC * C, 64) &&
              tc::make_map_2d_bf16(&mp.W, w.W, DK, NC * C, 64) && tc::make_map_2d_bf16(&mp.Ut, w.Ut, DV, NC * C, 64) &&
              tc::make_map_2d_bf16(&mp.T, w.Tn, C, NC * C, 64) && tc::make_map_2d_bf16(&mp.M, w.KK, C, NC * C, 64);
    if (ok) ok = t.dout && tc::make_map_4d_bf16(&mp.dout, t.dout, DV, H, T, Bn, 64);  // the backward requires dO
    if (!ok) return cudaErrorInvalidValue;
    Args a;
    a.beta = (const __nv_bfloat16 *)t.beta;
    a.dq = (__nv_bfloat16 *)t.dq; a.dk = (__nv_bfloat16 *)t.dk; a.dv = (__nv_bfloat16 *)t.dv;
    a.dalpha = (__nv_bfloat16 *)t.dalpha; a.dbeta = (__nv_bfloat16 *)t.dbeta; a.kwide = w.kwide;
    a.T = g.T; a.H = g.H; a.N = g.N; a.m0 = w.m0; a.m1 = w.m1;
    const size_t smem = SMEM_BYTES + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_bwd_kda_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    rec.mark(s);
    const uint64_t nrange = (uint64_t)g.B * g.H * ((w.m1 > 0 ? w.m1 : g.N) - w.m0);
    k_bwd_kda_tc<<<(unsigned)nrange, NTHREADS, smem, s>>>(mp, a);
    return cudaGetLastError();
}

}  // namespace dr
