// tc_bwd.cu -- all intra-chunk gradients of the backward on tcgen05 (Gated DeltaNet, DeltaNet).
//
// Backward of the chunked form of "线性注意力架构演进与Kimi Delta Attention创新实践"
// (sections 2.1, 6.2, 7.1) for one chunk of one (b, h), scalar gates.  With g the in-chunk
// cumulative log gate, E_ri = e^{g_r - g_i} (i <= r), S = S_n, dS+ = dL/dS_{n+1} and
// dU = du + P^T dO + Kbar dS+ (both from the reverse chain), and W, U~, U, P, T = (I+A)^-1,
// KK = k k^T, A = diag(beta) (KK .* E) from the recompute:
//
//   dP   = tril(dO U^T)                        dW = -dU S^T
//   dB_k = T^T dW,  dB_v = T^T dU              (through W = T diag(beta e^g) k, U~ = T diag(beta) v)
//   dA   = -strict_tril(dB_k W^T + dB_v U~^T)
//   D_P  = dP .* E,  D_M = diag(beta) dA .* E
//   dq   = diag(e^g) dO S^T + D_P k
//   dk   = D_P^T q + (D_M + D_M^T) k + diag(beta e^g) dB_k + Ubar dS+^T,   Ubar = diag(e^{g_C - g}) U
//   dv   = diag(beta) dB_v
//   dbeta_r = (dA .* KK .* E)_r. + e^{g_r} k_r . dB_k,r + v_r . dB_v,r
//   dg_r = e^{g_r} q_r . (dO S^T)_r + rowsum_r(Z) - colsum_r(Z) + beta_r e^{g_r} k_r . dB_k,r
//          - U_r . (Kbar dS+)_r,   Z = dP .* P + dA .* A,
//   dg_C += sum_r U_r . (Kbar dS+)_r + e^{g_C} sum(S .* dS+);
//   d log alpha = reverse cumulative sum of dg over the chunk.
// The row sums U_r . (Kbar dS+)_r come from the reverse chain, which forms Kbar dS+.
//
// Every product is token-major (rows = the chunk's 64 tokens), so that each gradient row and
// each per-token sum belongs to one thread: M = 128 MMAs whose rows 64..127 are discarded,
// except [dO ; dU] S^T, which stacks dq's dO S^T (rows 0-63) and dW (rows 64-127).  D_M + D_M^T
// needs no transpose: one D_M tile is read as a K-major and as an MN-major A operand.
//
// A persistent grid (one CTA of 256 threads per SM) walks the chunks.  Operands arrive by
// TMA in three groups (what the first products read; the rest; W and U~ into the space dO
// and dU leave), and the next chunk's first group is fetched into each of its regions as
// soon as the current chunk has finished with it; dq, dk, dv leave through staging tiles
// and TMA stores.  Warps w and w + 4 read the same TMEM lanes and split
// the columns; the warps of lanes 64-127 form dW and the sum of S .* dS+.  As in the
// per-chunk kernel, e^{g_r - g_i} is split at the chunk midpoint g_m unless the chunk's
// cumulative log gate strays more than 80 from it.
#include "tc_host.cuh"
#include "tc_inverse.cuh"
#include "tc_path.cuh"
#include "tc_ptx.cuh"
#include "tc_tile.cuh"

namespace dr {
namespace tcb {

using namespace dr::tc;
using dr::tcf::ld_chunk;
using dr::tcf::st_chunk;
using dr::tcf::tmem_row64;

constexpr int C = 64, DK = 128, DV = 128;
constexpr int NTHREADS = 256;
// shared memory (bytes from a 1024-aligned base); later phases reuse earlier regions
constexpr uint32_t R_DOU = 0;         // 32K  [dO_p0 | dU_p0 | dO_p1 | dU_p1], [r][j]  -> W [i][c] | U~ [i][j]
constexpr uint32_t R_S = 32768;       // 32K  S [c][j]
constexpr uint32_t R_DS = 65536;      // 32K  dS+ [c][j]
constexpr uint32_t R_U = 98304;       // 16K  U [r][j]  -> Ubar
constexpr uint32_t R_T = 114688;      //  8K  T [r][i]  -> D_M [r][i]
constexpr uint32_t R_P = 122880;      //  8K  P [r][i]  -> D_P [r][i]
constexpr uint32_t R_KK = 131072;     //  8K  KK [r][i]
constexpr uint32_t R_Q = 139264;      // 16K  q [r][c]
constexpr uint32_t R_K = 155648;      // 16K  k [r][c]
constexpr uint32_t R_V = 172032;      // 16K  v [r][j]  -> staging dv
constexpr uint32_t R_DW = 188416;     // 16K  dW [r][c] -> dB_k [r][c] -> fp32 dA' -> staging dq [r][c]
constexpr uint32_t R_BV = 204800;     // 16K  dB_v [r][j] -> fp32 dP -> staging dk [r][c]
constexpr uint32_t R_MISC = 221184;   //  8K
constexpr uint32_t SMEM_BYTES = R_MISC + 8192;
constexpr uint32_t LOAD1_BYTES = 4 * 16384 + 16384 + 512;             // dO, dU, S, U, g|beta
constexpr uint32_t LOAD2_BYTES = 32768 + 3 * 8192 + 3 * 16384 + 512;  // dS+, T, P, KK, q, k, v, row sums
constexpr uint32_t LOAD3_BYTES = 32768;                               // W, U~ (after batch 3)
// misc (floats unless noted)
constexpr uint32_t M_BAR = 0;  // [0] MMA, [1..3] load groups
constexpr uint32_t M_TMEM = 64, M_ABORT = 68;
constexpr uint32_t M_GB = 256;     // [2 chunks][2][64] g, beta   (bulk copies; this chunk's and the next's)
constexpr uint32_t M_SKT = 1280;   // [2][64] U . (Kbar dS+) per dv half (bulk copy)
constexpr uint32_t M_EG = 1792, M_EGC = 2048;  // [64] e^g, e^{g_C - g}
constexpr uint32_t M_PART = 2304;  // [3 kinds][2 column halves][64] per-row partial sums
constexpr uint32_t M_ROWQ = M_PART + 3 * 2 * 64 * 4;  // [rowsum Z, dbeta (A part)][4 column groups][64]
constexpr uint32_t M_ZC = M_ROWQ + 2 * 4 * 64 * 4;    // [2 row halves][64] column sums of Z
constexpr uint32_t M_RS = M_ZC + 512;               // [8] partial sums of S .* dS+
constexpr uint32_t M_DG = M_RS + 64;                // [64] dg, then [64] row sums
constexpr uint32_t M_ROWF = M_DG + 512, M_COLF = M_ROWF + 256;  // [64] e^{g_r - g_m}, e^{g_m - g_i}
constexpr uint32_t M_BIG = M_COLF + 256;            // int: the chunk's gate range needs exact exponentials
static_assert(M_BIG + 16 <= 8192, "misc overflow");
enum { PS_SQ = 0, PS_SBK, PS_SV, PS_NUM };
// TMEM columns
constexpr uint32_t TM_QW = 0;     // 128: rows 0-63 dO S^T, rows 64-127 dU S^T
constexpr uint32_t TM_X = 128;    // 128: dB_v, then D_P k
constexpr uint32_t TM_DP = 256;   //  64: dP
constexpr uint32_t TM_DA = 320;   //  64: dA'
constexpr uint32_t TM_DK = 256;   // 128: dk (after dP, dA' are consumed)
constexpr uint32_t TM_DBK = 384;  // 128: dB_k
constexpr uint32_t TM_COLS = 512;

struct Maps {
    CUtensorMap q, k, v, dout, dq, dk, dv;  // [B, T, H, 128] bf16; box 64 channels x 64 tokens
    CUtensorMap S, dS;                      // [chunks * 128][128] bf16; box 64 x 128
    CUtensorMap U, dU, W, Ut;               // [chunks * 64][128] bf16; box 64 x 64
    CUtensorMap P, T, KK;                   // [chunks * 64][64] bf16; box 64 x 64
};

struct Args {
    void *dalpha, *dbeta;  // bf16 [B, T, H]
    const float *gb;       // [chunks][2][64]: g, beta
    const float *skt;      // [chunks][2][64]
    int B, T, H, N, variant;    int m0, m1;            // the chunks [m0, m1) of each sequence (m1 = 0: all)
};

__device__ __forceinline__ void st_bf(void *p, size_t i, float x) {
    reinterpret_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(x);
}

// 32 fp32 columns of this thread's TMEM lane
__device__ __forceinline__ void tmem_row32(uint32_t taddr, float *v) {
    tmem_ld16(taddr + 0, v);
    tmem_ld16(taddr + 16, v + 16);
    wait_ld();
}

// v[t] (t = 0..15) held by every lane; returns, in the even lanes, the sum over the warp's 32
// lanes of v[lane >> 1] (butterfly transpose over four steps, then the pair of lanes).
__device__ __forceinline__ float warp_colsum16(float *v, int lane) {
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        const int m = 16 >> s, cnt = 8 >> s;
        const bool up = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < cnt; ++i) {
            const float lo = v[i], hi = v[i + cnt];
            const float send = up ? lo : hi;
            v[i] = (up ? hi : lo) + __shfl_xor_sync(0xffffffffu, send, m);
        }
    }
    return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
}

__global__ void __launch_bounds__(NTHREADS, 1) k_bwd_chunk_tc(const __grid_constant__ Maps mp, Args a) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    unsigned char *misc = sm + R_MISC;
    uint64_t *bar = reinterpret_cast<uint64_t *>(misc + M_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + M_TMEM);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + M_ABORT);
    const float *skt = reinterpret_cast<const float *>(misc + M_SKT);
    float *eg = reinterpret_cast<float *>(misc + M_EG);
    float *egc = reinterpret_cast<float *>(misc + M_EGC);
    float *part = reinterpret_cast<float *>(misc + M_PART);
    float *zc = reinterpret_cast<float *>(misc + M_ZC);
    float *rowq = reinterpret_cast<float *>(misc + M_ROWQ);
    float *rsp = reinterpret_cast<float *>(misc + M_RS);
    float *dgs = reinterpret_cast<float *>(misc + M_DG);
    float *ktm = dgs + 64;
    float *rowf = reinterpret_cast<float *>(misc + M_ROWF);
    float *colf = reinterpret_cast<float *>(misc + M_COLF);
    volatile int *bigflag = reinterpret_cast<volatile int *>(misc + M_BIG);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q4 = warp & 3, hf = warp >> 2;
    const bool rowt = q4 < 2;            // owns token row r of the accumulators
    const int r = (q4 & 1) * 32 + lane;  // token row (TMEM rows 64 + r for q4 >= 2)
    const int T = a.T, H = a.H, N = a.N, m0 = a.m0, NS = (a.m1 > 0 ? a.m1 : N) - m0, total = a.B * H * NS;
    const bool gated = a.variant == VAR_GATED;
    auto part_at = [&](int kind, int half, int rr) -> float & { return part[(kind * 2 + half) * 64 + rr]; };
    struct Pos { int ci, n, h, b, t0; };
    // work item wi: chunk n = m0 + wi / (B H) of sequence (b, h) = wi % (B H), chunk by chunk from the
    // first: the reverse chain wrote the first chunks' dS and dU last, so they are read while in L2
    const int BH = a.B * H;
    auto pos_of = [&](int wi) -> Pos {
        Pos p;
        p.n = m0 + wi / BH;
        const int bh = wi % BH;
        p.ci = bh * N + p.n;
        p.h = bh % H; p.b = bh / H; p.t0 = p.n * C;
        return p;
    };
    // the first load group of a chunk: dO, dU, S, U, g|beta (issued in three parts for the next chunk)
    auto load1_s = [&](const Pos &p, int gbuf) {
#pragma unroll
        for (int q = 0; q < 2; ++q) tma_load_2d(sm + R_S + q * 16384, &mp.S, 64 * q, p.ci * DK, &bar[1]);
        bulk_load(misc + M_GB + gbuf * 512, a.gb + (size_t)p.ci * 2 * C, 512, &bar[1]);
    };
    auto load1_dou = [&](const Pos &p) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            tma_load_4d(sm + R_DOU + q * 16384, &mp.dout, 64 * q, p.h, p.t0, p.b, &bar[1]);
            tma_load_2d(sm + R_DOU + q * 16384 + 8192, &mp.dU, 64 * q, p.ci * C, &bar[1]);
        }
    };
    auto load1_u = [&](const Pos &p) {
#pragma unroll
        for (int q = 0; q < 2; ++q) tma_load_2d(sm + R_U + q * 8192, &mp.U, 64 * q, p.ci * C, &bar[1]);
    };

    // issue state of thread 0 (the only thread that issues TMA and MMA): phases armed per barrier
    int armed[4] = {0, 0, 0, 0};
    if (tid == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(&bar[i], 1);
        *abort_flag = 0;
        fence_mbar_init();
        if ((int)blockIdx.x < total) {
            const Pos p0 = pos_of(blockIdx.x);
            mbar_arrive_tx(&bar[1], LOAD1_BYTES);
            load1_s(p0, 0);
            load1_dou(p0);
            load1_u(p0);
            armed[1] = 1;
        }
    }
    if (warp == 0) tmem_alloc(tmem_slot, TM_COLS);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tl = tbase + ((uint32_t)(q4 * 32) << 16);
    uint32_t ph = 0;
    auto consensus = [&](bool ok) -> bool { return !named_sync_any(1, NTHREADS, !ok || *abort_flag != 0); };
    auto commit_mma = [&]() {
        mma_commit(&bar[0]);
        armed[0]++;
    };
    auto wait_mma = [&]() -> bool {
        const bool ok = mbar_wait(&bar[0], ph & 1, abort_flag);
        ph++;
        fence_after_sync();
        return consensus(ok);
    };
    const uint32_t sDOU = smem_u32(sm + R_DOU), sS = smem_u32(sm + R_S), sDS = smem_u32(sm + R_DS);
    const uint32_t sU = smem_u32(sm + R_U), sT = smem_u32(sm + R_T), sP = smem_u32(sm + R_P);
    const uint32_t sQ = smem_u32(sm + R_Q), sK = smem_u32(sm + R_K), sDW = smem_u32(sm + R_DW);
    const uint32_t sBV = smem_u32(sm + R_BV);

    bool ok = true;
    int it = 0;
    for (int cidx = blockIdx.x; cidx < total && ok; cidx += gridDim.x, ++it) {
        const Pos p = pos_of(cidx);
        const int ci = p.ci, h = p.h, b = p.b, t0 = p.t0, L = min(C, T - t0);
        const int cnext = cidx + (int)gridDim.x;
        const bool has_next = cnext < total;
        const Pos pn = pos_of(has_next ? cnext : cidx);
        const float *gsm = reinterpret_cast<const float *>(misc + M_GB + (it & 1) * 512);  // g [64], beta [64]
        auto trow_g = [&](int rr) -> size_t { return ((size_t)b * T + t0 + rr) * H + h; };  // token row (rr < L)

        // second load group of this chunk (its regions were released by the previous chunk,
        // once the previous chunk's stores have read their staging tiles)
        if (tid == 0) {
            bulk_wait_read_all();
            mbar_arrive_tx(&bar[2], LOAD2_BYTES);
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                tma_load_2d(sm + R_DS + q * 16384, &mp.dS, 64 * q, ci * DK, &bar[2]);
                tma_load_4d(sm + R_Q + q * 8192, &mp.q, 64 * q, h, t0, b, &bar[2]);
                tma_load_4d(sm + R_K + q * 8192, &mp.k, 64 * q, h, t0, b, &bar[2]);
                tma_load_4d(sm + R_V + q * 8192, &mp.v, 64 * q, h, t0, b, &bar[2]);
            }
            tma_load_2d(sm + R_T, &mp.T, 0, ci * C, &bar[2]);
            tma_load_2d(sm + R_P, &mp.P, 0, ci * C, &bar[2]);
            tma_load_2d(sm + R_KK, &mp.KK, 0, ci * C, &bar[2]);
            bulk_load(misc + M_SKT, a.skt + (size_t)ci * 2 * C, 512, &bar[2]);
            armed[2]++;
        }
        ok = consensus(mbar_wait(&bar[1], it & 1, abort_flag));
        if (!ok) break;
        // ---------------- batch 1: [dO ; dU] S^T, dP = dO U^T ----------------
        if (tid == 0) {
            const uint32_t id_qw = idesc_bf16(128, 128, 0, 0), id_p = idesc_bf16(128, 64, 0, 0);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t ka = (k >> 2) * 16384 + (k & 3) * 32;
                mma_bf16(tbase + TM_QW, sdesc(sDOU + ka, 16, 1024), sdesc(sS + ka, 16, 1024), id_qw, k > 0);
                mma_bf16(tbase + TM_DP, sdesc(sDOU + ka, 16, 1024),
                         sdesc(sU + (k >> 2) * 8192 + (k & 3) * 32, 16, 1024), id_p, k > 0);
            }
            commit_mma();
        }
        // gate factors
        if (tid < C) {
            const float x = gsm[tid], gm = gsm[31];
            eg[tid] = __expf(x);
            egc[tid] = __expf(gsm[C - 1] - x);
            rowf[tid] = __expf(x - gm);
            colf[tid] = __expf(gm - x);
            const float dev = warp_max(fabsf(x - gm));
            if (lane == 0 && warp == 0) *bigflag = 0;
            named_sync(3, 64);
            if (lane == 0 && dev > 80.f) *bigflag = 1;
        }
        ok = wait_mma();
        if (!ok) break;
        // ---------------- epilogue 1: dW = -(dU S^T) -> tile;  Ubar = diag(e^{gC - g}) U ----------------
        if (!rowt) {
            float v[64];
            tmem_row64(tl + TM_QW + hf * 64, v);
#pragma unroll
            for (int j = 0; j < 64; ++j) v[j] = -v[j];
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) st_chunk(sm + R_DW, (uint32_t)hf * 8192 + swz(r, ch), v + ch * 8);
        } else {
            const float f = egc[r];
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                const uint32_t o = (uint32_t)hf * 8192 + swz(r, ch);
                float v[8];
                ld_chunk(sm + R_U, o, v);
#pragma unroll
                for (int e = 0; e < 8; ++e) v[e] *= f;
                st_chunk(sm + R_U, o, v);
            }
        }
        fence_proxy_async();
        fence_before_sync();
        ok = consensus(mbar_wait(&bar[2], it & 1, abort_flag));  // T, k, v, ...
        if (!ok) break;
        // ---------------- batch 3: dB_k = T^T dW, dB_v = T^T dU ----------------
        if (tid == 0) {
            fence_after_sync();
            const uint32_t id = idesc_bf16(128, 128, 1, 1);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                mma_bf16(tbase + TM_DBK, sdesc(sT + k * 2048, 8192, 1024), sdesc(sDW + k * 2048, 8192, 1024), id,
                         k > 0);
                mma_bf16(tbase + TM_X, sdesc(sT + k * 2048, 8192, 1024), sdesc(sDOU + 8192 + k * 2048, 16384, 1024),
                         id, k > 0);
            }
            commit_mma();
        }
        ok = wait_mma();
        if (!ok) break;
        // third load group into the space dO and dU leave
        if (tid == 0) {
            mbar_arrive_tx(&bar[3], LOAD3_BYTES);
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                tma_load_2d(sm + R_DOU + q * 8192, &mp.W, 64 * q, ci * C, &bar[3]);
                tma_load_2d(sm + R_DOU + 16384 + q * 8192, &mp.Ut, 64 * q, ci * C, &bar[3]);
            }
            armed[3]++;
        }
        // the sum of S .* dS+ (lanes 64-127, idle in this epilogue)
        if (!rowt) {
            float rs = 0.f;
            for (int x = (q4 - 2) * 32 + lane + hf * 64; x < 2048; x += 128) {  // S, dS+: one layout
                float v[8], w[8];
                ld_chunk(sm + R_S, (uint32_t)x * 16, v);
                ld_chunk(sm + R_DS, (uint32_t)x * 16, w);
#pragma unroll
                for (int e = 0; e < 8; ++e) rs += v[e] * w[e];
            }
            rs = warp_sum(rs);
            if (lane == 0) rsp[warp] = rs;
        }
        // ---------------- epilogue 3: dB_k, dB_v tiles; dv; dbeta sums ----------------
        if (rowt) {
            float x[64];
            float sbk = 0.f, sv = 0.f;
            tmem_row64(tl + TM_DBK + hf * 64, x);
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                const uint32_t o = (uint32_t)hf * 8192 + swz(r, ch);
                float kv[8];
                ld_chunk(sm + R_K, o, kv);
#pragma unroll
                for (int e = 0; e < 8; ++e) sbk += kv[e] * x[ch * 8 + e];
                st_chunk(sm + R_DW, o, x + ch * 8);
            }
            tmem_row64(tl + TM_X + hf * 64, x);
            const float br = gsm[C + r];
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                const uint32_t o = (uint32_t)hf * 8192 + swz(r, ch);
                float vv[8];
                ld_chunk(sm + R_V, o, vv);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    sv += vv[e] * x[ch * 8 + e];
                    vv[e] = br * x[ch * 8 + e];
                }
                st_chunk(sm + R_BV, o, x + ch * 8);
                st_chunk(sm + R_V, o, vv);  // dv, in place of v
            }
            part_at(PS_SBK, hf, r) = sbk;
            part_at(PS_SV, hf, r) = sv;
        }
        fence_proxy_async();
        fence_before_sync();
        ok = consensus(true);
        if (!ok) break;
        if (tid == 0) {
            fence_after_sync();
            tma_store_4d(&mp.dv, sm + R_V, 0, h, t0, b);
            tma_store_4d(&mp.dv, sm + R_V + 8192, 64, h, t0, b);
            bulk_commit();
            if (has_next) {  // the next chunk's S (and g, beta) into the space S leaves
                mbar_arrive_tx(&bar[1], LOAD1_BYTES);
                load1_s(pn, (it + 1) & 1);
                armed[1]++;
            }
        }
        ok = consensus(mbar_wait(&bar[3], it & 1, abort_flag));  // W, U~
        if (!ok) break;
        // ---------------- batch 4: dA' = dB_k W^T + dB_v U~^T ----------------
        if (tid == 0) {
            fence_after_sync();
            const uint32_t id = idesc_bf16(128, 64, 0, 0);
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const uint32_t ka = ((k & 7) >> 2) * 8192 + (k & 3) * 32;
                const uint32_t aa = (k < 8 ? sDW : sBV) + ka, bb = sDOU + (k < 8 ? 0 : 16384) + ka;
                mma_bf16(tbase + TM_DA, sdesc(aa, 16, 1024), sdesc(bb, 16, 1024), id, k > 0);
            }
            commit_mma();
        }
        ok = wait_mma();
        if (!ok) break;
        if (tid == 0 && has_next) load1_dou(pn);  // the next chunk's dO, dU into the space W, U~ leave
        // ---------------- epilogue 4: D_P, D_M, Z, dbeta (A part) ----------------
        // Lanes 0-63 copy dA' and dP (fp32) into the dB tiles batch 4 has finished reading; then
        // every thread takes 16 columns of one row (all four SM sub-partitions share the work).
        float *daf = reinterpret_cast<float *>(sm + R_DW), *dpf = reinterpret_cast<float *>(sm + R_BV);
        if (rowt) {
            float da[32], dp[32];
            tmem_row32(tl + TM_DA + hf * 32, da);
            tmem_row32(tl + TM_DP + hf * 32, dp);
#pragma unroll
            for (int c4 = 0; c4 < 8; ++c4) {
                const int o = sw64(r, hf * 32 + c4 * 4);
                *reinterpret_cast<float4 *>(daf + o) =
                    make_float4(da[4 * c4], da[4 * c4 + 1], da[4 * c4 + 2], da[4 * c4 + 3]);
                *reinterpret_cast<float4 *>(dpf + o) =
                    make_float4(dp[4 * c4], dp[4 * c4 + 1], dp[4 * c4 + 2], dp[4 * c4 + 3]);
            }
        }
        ok = consensus(true);
        if (!ok) break;
        {
            const int rr = tid & 63, cg = tid >> 6, c0 = cg * 16;  // row, 16-column group
            float da[16], dp[16], pv[16], kk[16];
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                const int o = sw64(rr, c0 + c4 * 4);
                const float4 x = *reinterpret_cast<const float4 *>(daf + o);
                const float4 y = *reinterpret_cast<const float4 *>(dpf + o);
                da[4 * c4] = x.x; da[4 * c4 + 1] = x.y; da[4 * c4 + 2] = x.z; da[4 * c4 + 3] = x.w;
                dp[4 * c4] = y.x; dp[4 * c4 + 1] = y.y; dp[4 * c4 + 2] = y.z; dp[4 * c4 + 3] = y.w;
            }
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
                ld_chunk(sm + R_P, swz(rr, cg * 2 + c2), pv + c2 * 8);
                ld_chunk(sm + R_KK, swz(rr, cg * 2 + c2), kk + c2 * 8);
            }
            const float br = gsm[C + rr], gr = gsm[rr];
            // gate factor e^{g_r - g_i}: 1 without gates, else split at the midpoint unless the range is large
            float ef[16];
            if (!gated) {
#pragma unroll
                for (int t = 0; t < 16; ++t) ef[t] = 1.f;
            } else if (*bigflag == 0) {
                const float rf = rowf[rr];
#pragma unroll
                for (int t = 0; t < 16; ++t) ef[t] = rf * colf[c0 + t];
            } else {
#pragma unroll
                for (int t = 0; t < 16; ++t) ef[t] = __expf(gr - gsm[c0 + t]);
            }
            float rowz = 0.f, dbA = 0.f;
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                const int i = c0 + t;
                const float e = (i <= rr) ? ef[t] : 0.f;
                const float d = (i < rr) ? -da[t] : 0.f;
                const float pp = (i <= rr) ? dp[t] : 0.f;
                const float dak = d * kk[t] * e;
                dbA += dak;
                const float z = pp * pv[t] + br * dak;
                rowz += z;
                dp[t] = pp * e;      // D_P
                da[t] = br * d * e;  // D_M
                pv[t] = z;
            }
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
                st_chunk(sm + R_P, swz(rr, cg * 2 + c2), dp + c2 * 8);
                st_chunk(sm + R_T, swz(rr, cg * 2 + c2), da + c2 * 8);
            }
            rowq[(0 * 4 + cg) * 64 + rr] = rowz;
            rowq[(1 * 4 + cg) * 64 + rr] = dbA;
            const float zsum = warp_colsum16(pv, lane);
            if ((lane & 1) == 0) zc[(warp & 1) * 64 + c0 + (lane >> 1)] = zsum;
        }
        fence_proxy_async();
        fence_before_sync();
        ok = consensus(true);
        if (!ok) break;
        // ---------------- batch 5: D_P k;  dk = D_P^T q + D_M k + D_M^T k + Ubar dS+^T ----------------
        if (tid == 0) {
            fence_after_sync();
            const uint32_t id_km = idesc_bf16(128, 128, 0, 1), id_mm = idesc_bf16(128, 128, 1, 1);
            const uint32_t id_kk = idesc_bf16(128, 128, 0, 0);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                mma_bf16(tbase + TM_X, sdesc(sP + k * 32, 16, 1024), sdesc(sK + k * 2048, 8192, 1024), id_km, k > 0);
                mma_bf16(tbase + TM_DK, sdesc(sP + k * 2048, 8192, 1024), sdesc(sQ + k * 2048, 8192, 1024), id_mm,
                         k > 0);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                mma_bf16(tbase + TM_DK, sdesc(sT + k * 32, 16, 1024), sdesc(sK + k * 2048, 8192, 1024), id_km, 1);
                mma_bf16(tbase + TM_DK, sdesc(sT + k * 2048, 8192, 1024), sdesc(sK + k * 2048, 8192, 1024), id_mm, 1);
            }
#pragma unroll
            for (int k = 0; k < 8; ++k)
                mma_bf16(tbase + TM_DK, sdesc(sU + (k >> 2) * 8192 + (k & 3) * 32, 16, 1024),
                         sdesc(sDS + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024), id_kk, 1);
            commit_mma();
        }
        ok = wait_mma();
        if (!ok) break;
        if (tid == 0 && has_next) load1_u(pn);  // the next chunk's U into the space Ubar leaves
        // ---------------- epilogue 5: dq, dk rows (staged in the dB tiles); e^g q . (dO S^T) ----------------
        if (rowt) {
            const float er = eg[r], bk = gsm[C + r] * er;
            float x[64], y[64];
            float sq = 0.f;
            tmem_row64(tl + TM_QW + hf * 64, x);  // dO S^T
            tmem_row64(tl + TM_X + hf * 64, y);   // D_P k
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                const uint32_t o = (uint32_t)hf * 8192 + swz(r, ch);
                float qv[8], w[8];
                ld_chunk(sm + R_Q, o, qv);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    sq += qv[e] * x[ch * 8 + e];
                    w[e] = er * x[ch * 8 + e] + y[ch * 8 + e];
                }
                st_chunk(sm + R_DW, o, w);
            }
            part_at(PS_SQ, hf, r) = er * sq;
            tmem_row64(tl + TM_DK + hf * 64, x);
            tmem_row64(tl + TM_DBK + hf * 64, y);
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                float w[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) w[e] = x[ch * 8 + e] + bk * y[ch * 8 + e];
                st_chunk(sm + R_BV, (uint32_t)hf * 8192 + swz(r, ch), w);
            }
        }
        fence_proxy_async();
        fence_before_sync();
        ok = consensus(true);
        if (!ok) break;
        if (tid == 0) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                tma_store_4d(&mp.dq, sm + R_DW + q * 8192, 64 * q, h, t0, b);
                tma_store_4d(&mp.dk, sm + R_BV + q * 8192, 64 * q, h, t0, b);
            }
            bulk_commit();
        }
        // ---------------- dbeta, dg, d log alpha ----------------
        if (tid < C) {
            const int rr = tid;
            const float sq = part_at(PS_SQ, 0, rr) + part_at(PS_SQ, 1, rr);
            const float sbk = eg[rr] * (part_at(PS_SBK, 0, rr) + part_at(PS_SBK, 1, rr));
            const float sv = part_at(PS_SV, 0, rr) + part_at(PS_SV, 1, rr);
            const float rowz = rowq[rr] + rowq[64 + rr] + rowq[128 + rr] + rowq[192 + rr];
            const float dbA = rowq[256 + rr] + rowq[320 + rr] + rowq[384 + rr] + rowq[448 + rr];
            const float zcol = zc[rr] + zc[64 + rr];
            const float sk = skt[rr] + skt[C + rr];
            if (rr < L) st_bf(a.dbeta, trow_g(rr), dbA + sbk + sv);
            dgs[rr] = rowz - zcol + sq + gsm[C + rr] * sbk - sk;
            ktm[rr] = sk;
        }
        ok = consensus(true);
        if (!ok) break;
        if (gated && warp == 0) {
            const float a0 = dgs[2 * lane];
            float a1 = dgs[2 * lane + 1];
            const float tsum = warp_sum(ktm[2 * lane] + ktm[2 * lane + 1]);
            const float rs = rsp[2] + rsp[3] + rsp[6] + rsp[7];
            // the chunk-end terms belong to dg_C (last row): the U . (Kbar dS+) sums and the decay
            // e^{g_C} of the incoming state
            if (lane == 31) a1 += tsum + __expf(gsm[C - 1]) * rs;
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
        // the misc scratch and the gate factors are rewritten by the next chunk
        ok = consensus(true);
    }
    if (tid == 0) {
        bulk_wait_all();
        if (*abort_flag) {  // let whatever was issued finish before the CTA leaves
            volatile int dummy = 0;
            for (int i = 0; i < 4; ++i)
                if (armed[i] > 0) mbar_wait(&bar[i], (armed[i] - 1) & 1, &dummy, 100000000ull);
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
    const bool ok =
        tc::make_map_4d_bf16(&mp.q, t.q, DK, H, T, Bn, 64) && tc::make_map_4d_bf16(&mp.k, t.k, DK, H, T, Bn, 64) &&
        tc::make_map_4d_bf16(&mp.v, t.v, DV, H, T, Bn, 64) && tc::make_map_4d_bf16(&mp.dout, t.dout, DV, H, T, Bn, 64) &&
        tc::make_map_4d_bf16(&mp.dq, t.dq, DK, H, T, Bn, 64) && tc::make_map_4d_bf16(&mp.dk, t.dk, DK, H, T, Bn, 64) &&
        tc::make_map_4d_bf16(&mp.dv, t.dv, DV, H, T, Bn, 64) && tc::make_map_2d_bf16(&mp.S, w.Sn, DV, NC * DK, 128) &&
        tc::make_map_2d_bf16(&mp.dS, w.dSn, DV, NC * DK, 128) && tc::make_map_2d_bf16(&mp.U, w.Un, DV, NC * C, 64) &&
        tc::make_map_2d_bf16(&mp.dU, w.dUn, DV, NC * C, 64) && tc::make_map_2d_bf16(&mp.W, w.W, DK, NC * C, 64) &&
        tc::make_map_2d_bf16(&mp.Ut, w.Ut, DV, NC * C, 64) && tc::make_map_2d_bf16(&mp.P, w.P, C, NC * C, 64) &&
        tc::make_map_2d_bf16(&mp.T, w.Tn, C, NC * C, 64) && tc::make_map_2d_bf16(&mp.KK, w.KK, C, NC * C, 64);
    if (!ok) return cudaErrorInvalidValue;
    Args a;
    a.dalpha = t.dalpha; a.dbeta = t.dbeta; a.gb = w.gb; a.skt = w.skt;
    a.B = g.B; a.T = g.T; a.H = g.H; a.N = g.N; a.variant = g.variant; a.m0 = w.m0; a.m1 = w.m1;
    const size_t smem = SMEM_BYTES + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_bwd_chunk_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    rec.mark(s);
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const long long total = (long long)g.B * g.H * ((w.m1 > 0 ? w.m1 : g.N) - w.m0);
    const int grid = (int)(total < sms ? total : sms);
    k_bwd_chunk_tc<<<grid, NTHREADS, smem, s>>>(mp, a);
    return cudaGetLastError();
}

}  // namespace dr
