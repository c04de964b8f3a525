// tc_state.cu -- the backward's products with the chunk states on tcgen05, for the KDA backward.
//
// For one chunk of one (b, h), with S = S_n (the state entering the chunk), dS+ = dL/dS_{n+1},
// U the chunk's write values, dU = dL/dU (both from the reverse chain) and dO the output
// gradient, the intra-chunk gradient needs (chunked form of "线性注意力架构演进与Kimi Delta
// Attention创新实践", sections 2.1 and 6.2; no gate enters these four):
//   Qd = dO S^T,   dWm = -dU S^T,   Tm = U dS+^T   ([64][dk] each),   RS = rowsum(S .* dS+)  ([dk])
// One CTA of 128 threads per chunk.  TMA brings S, dS+ ([128][128] each), dO and dU (stacked as
// one [128][128] operand) and U ([64][128]) as bf16 128-byte-swizzled tiles; two MMAs with the
// state as the 128-row operand give the transposed products in TMEM,
//   D1 = S [dO ; dU]^T  (lane c, columns 0-63: Qd[.][c], 64-127: -dWm[.][c]),
//   D2 = dS+ U^T        (lane c, columns 128-191: Tm[.][c]),
// so that thread c writes column c of each result: every warp store covers 32 consecutive
// channels.  RS comes from the same tiles in shared memory.  The results go to the fp32
// workspace of the CUDA-core intra-chunk gradient kernel, in place of its CUDA-core products
// (which read the same bf16 values widened to fp32, so only the summation order differs).
#include "tc_host.cuh"
#include "tc_path.cuh"
#include "tc_ptx.cuh"
#include "tc_tile.cuh"

namespace dr {
namespace tcs {

using namespace dr::tc;
using dr::tcf::ld_chunk;
using dr::tcf::tmem_row64;

constexpr int C = 64, DK = 128, DV = 128;
constexpr int NTHREADS = 128;
constexpr uint32_t R_S = 0;          // 32K  S [c][j]: two 64-column panels of 128 rows
constexpr uint32_t R_DS = 32768;     // 32K  dS+ [c][j]
constexpr uint32_t R_DOU = 65536;    // 32K  per panel: dO rows 0-63 (8K), then dU rows 64-127 (8K)
constexpr uint32_t R_U = 98304;      // 16K  U [r][j]: two panels of 64 rows
constexpr uint32_t R_MISC = 114688;  // barriers, TMEM slot, abort flag
constexpr uint32_t SMEM_BYTES = R_MISC + 64;
constexpr uint32_t TM_D1 = 0, TM_D2 = 128, TM_COLS = 256;

struct Maps {
    CUtensorMap S, dS, U, dU;  // workspace tiles, bf16
    CUtensorMap dout;          // [B, T, H, 128] bf16; box 64 channels x 64 tokens
};

struct Args {
    float *Qd, *dWm, *Tm, *RS;  // [ci][C][dk] x3, [ci][dk] (fp32)
    const int *only;            // optional: the chunks flagged here alone
    int has_dout, T, H, N;
};

__global__ void __launch_bounds__(NTHREADS, 1) k_state_tc(const __grid_constant__ Maps mp, Args a) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + R_MISC);  // [0] loads, [1] MMA
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + R_MISC + 16);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + R_MISC + 20);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int ci = blockIdx.x, n = ci % a.N, bh = ci / a.N, h = bh % a.H, b = bh / a.H, t0 = n * C;
    if (a.only && !a.only[ci]) return;  // uniform over the CTA
    const uint32_t load_bytes = 2 * 32768 + (a.has_dout ? 16384 : 0) + 16384 + 16384;
    if (!a.has_dout)  // no output gradient: the dO rows of the stacked operand are zero
        for (int x = tid; x < 2 * 8192 / 16; x += NTHREADS)
            *reinterpret_cast<uint4 *>(sm + R_DOU + (x >> 9) * 16384 + (x & 511) * 16) = make_uint4(0, 0, 0, 0);
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        *abort_flag = 0;
        fence_mbar_init();
        mbar_arrive_tx(&bar[0], load_bytes);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            tma_load_2d(sm + R_S + q * 16384, &mp.S, 64 * q, ci * DK, &bar[0]);
            tma_load_2d(sm + R_DS + q * 16384, &mp.dS, 64 * q, ci * DK, &bar[0]);
            if (a.has_dout) tma_load_4d(sm + R_DOU + q * 16384, &mp.dout, 64 * q, h, t0, b, &bar[0]);
            tma_load_2d(sm + R_DOU + q * 16384 + 8192, &mp.dU, 64 * q, ci * C, &bar[0]);
            tma_load_2d(sm + R_U + q * 8192, &mp.U, 64 * q, ci * C, &bar[0]);
        }
    }
    fence_proxy_async();  // the zeroed dO rows, for the MMA's reads
    if (warp == 0) tmem_alloc(tmem_slot, TM_COLS);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = *tmem_slot;
    bool ok = !named_sync_any(1, NTHREADS, !mbar_wait(&bar[0], 0, abort_flag) || *abort_flag != 0);
    bool mma_armed = false;
    if (ok && tid == 0) {
        const uint32_t sS = smem_u32(sm + R_S), sDS = smem_u32(sm + R_DS), sDOU = smem_u32(sm + R_DOU);
        const uint32_t sU = smem_u32(sm + R_U);
        const uint32_t id1 = idesc_bf16(128, 128, 0, 0), id2 = idesc_bf16(128, 64, 0, 0);
#pragma unroll
        for (int k = 0; k < 8; ++k) {  // K = dv in steps of 16
            const uint32_t ka = (k >> 2) * 16384 + (k & 3) * 32;
            mma_bf16(tbase + TM_D1, sdesc(sS + ka, 16, 1024), sdesc(sDOU + ka, 16, 1024), id1, k > 0);
            mma_bf16(tbase + TM_D2, sdesc(sDS + ka, 16, 1024), sdesc(sU + (k >> 2) * 8192 + (k & 3) * 32, 16, 1024),
                     id2, k > 0);
        }
        mma_commit(&bar[1]);
        mma_armed = true;
    }
    if (ok) {
        ok = !named_sync_any(1, NTHREADS, !mbar_wait(&bar[1], 0, abort_flag) || *abort_flag != 0);
        fence_after_sync();
    }
    if (ok) {
        const int c = tid;  // TMEM lane = key channel (warp w reads lanes 32 w .. 32 w + 31)
        const uint32_t tl = tbase + ((uint32_t)(warp * 32) << 16);
        const size_t base = (size_t)ci * C * DK + c;
        float v[64];
        tmem_row64(tl + TM_D1, v);
#pragma unroll
        for (int r = 0; r < C; ++r) a.Qd[base + (size_t)r * DK] = v[r];
        tmem_row64(tl + TM_D1 + 64, v);
#pragma unroll
        for (int r = 0; r < C; ++r) a.dWm[base + (size_t)r * DK] = -v[r];
        tmem_row64(tl + TM_D2, v);
#pragma unroll
        for (int r = 0; r < C; ++r) a.Tm[base + (size_t)r * DK] = v[r];
        float rs = 0.f;
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                float s8[8], d8[8];
                const uint32_t o = (uint32_t)q * 16384 + swz(c, ch);
                ld_chunk(sm + R_S, o, s8);
                ld_chunk(sm + R_DS, o, d8);
#pragma unroll
                for (int e = 0; e < 8; ++e) rs += s8[e] * d8[e];
            }
        a.RS[(size_t)ci * DK + c] = rs;
    }
    if (tid == 0 && !ok) {  // let whatever was issued land before the CTA leaves
        volatile int dummy = 0;
        mbar_wait(&bar[0], 0, &dummy, 100000000ull);
        if (mma_armed) mbar_wait(&bar[1], 0, &dummy, 100000000ull);
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == 0) tmem_dealloc(tbase, TM_COLS);
}

}  // namespace tcs

cudaError_t tc_state_to_simt(const Geo &g, const Tensors &t, const TcWs &w, float *Qd, float *dWm, float *Tm,
                             float *RS, cudaStream_t s, Rec &rec, const int *only) {
    using namespace tcs;
    Maps mp;
    const uint64_t Bn = g.B, T = g.T, H = g.H, NC = (uint64_t)g.B * g.H * g.N;
    bool ok = tc::make_map_2d_bf16(&mp.S, w.Sn, DV, NC * DK, 128) && tc::make_map_2d_bf16(&mp.dS, w.dSn, DV, NC * DK, 128) &&
              tc::make_map_2d_bf16(&mp.U, w.Un, DV, NC * C, 64) && tc::make_map_2d_bf16(&mp.dU, w.dUn, DV, NC * C, 64);
    if (ok && t.dout) ok = tc::make_map_4d_bf16(&mp.dout, t.dout, DV, H, T, Bn, 64);
    if (!ok) return cudaErrorInvalidValue;
    Args a;
    a.Qd = Qd; a.dWm = dWm; a.Tm = Tm; a.RS = RS; a.only = only;
    a.has_dout = t.dout != nullptr; a.T = g.T; a.H = g.H; a.N = g.N;
    const size_t smem = SMEM_BYTES + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_state_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    rec.mark(s);
    k_state_tc<<<(unsigned)NC, NTHREADS, smem, s>>>(mp, a);
    return cudaGetLastError();
}

}  // namespace dr
