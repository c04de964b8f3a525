// tc_bwd.cu -- per-chunk products of the backward with the chunk's states, on tcgen05.
//
// For one chunk of one (b, h), with S = S_n (state entering the chunk), dS+ = dL/dS_{n+1},
// U the write values, P = tril(Qtil Khat^T) and Kbar = e^{g_C - g} k (the chunk-end decay of
// each token), the backward of the chunked form of "线性注意力架构演进与Kimi Delta Attention
// 创新实践" (sections 2.1, 6.2) needs
//     dU  = du + P^T dO + Kbar dS+           (C x dv)  total gradient of the write values
//     Qd  = dO S^T,  dWm = -dU S^T,  Tm = U dS+^T     (C x dk each)
//     RS  = rowsum(S .* dS+)                 (dk)
// Every product is computed channel-major so that M = 128 (dk or dv) fills the MMA:
//     dU^T  = dO^T P + dS+^T Kbar^T          (A: MN-major dO, dS+; B: P MN-major, Kbar K-major)
//     Qd^T  = S dO^T,  Tm^T = dS+ U^T,  dWm^T = -S dU^T
// One CTA (128 threads) per chunk; operands are converted to bf16 in 128B-swizzled tiles.
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
// shared memory (bytes from a 1024-aligned base)
constexpr uint32_t OFF_S = 0;              // 32K  S        [c][j]  K-major, 2 panels of 16K
constexpr uint32_t OFF_DS = 32768;         // 32K  dS+      [c][j]
constexpr uint32_t OFF_U = 65536;          // 16K  U        [r][j]  2 panels of 8K
constexpr uint32_t OFF_DO = 81920;         // 16K  dO       [r][j]
constexpr uint32_t OFF_KB = 98304;         // 16K  Kbar     [r][c]
constexpr uint32_t OFF_P = 114688;         //  8K  P        [i][r]  (row-major P)
constexpr uint32_t OFF_DUT = 122880;       // 16K  dU^T     [j][r]
constexpr uint32_t OFF_MISC = 139264;      //  1K
constexpr uint32_t SMEM_BYTES = OFF_MISC + 1024;
constexpr uint32_t TM_DUT = 0, TM_QD = 64, TM_TM = 128, TM_DW = 192, TM_COLS = 256;

struct Args {
    const void *k, *dout, *du;  // bf16 [B,T,H,d]
    SimtWs w;
    int B, T, H, N;
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

__global__ void __launch_bounds__(NTHREADS, 1) k_bwd_state_tc(Args a) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + OFF_MISC);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC + 64);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + OFF_MISC + 68);
    const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int T = a.T, H = a.H, t0 = n * C, L = min(C, T - t0);
    const size_t ci = ((size_t)b * H + h) * a.N + n;

    if (tid == 0) {
        mbar_init(bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, TM_COLS);

    // ---- operands -> bf16 tiles ----
    const float *Sg = a.w.Sn + ci * DK * DV, *dSg = a.w.dSn + ci * DK * DV;
    for (int x = tid; x < DK * 16; x += NTHREADS) {   // S, dS+: 128 rows x 16 chunks
        const int r = x >> 4, c16 = x & 15, p = c16 >> 3, ch = c16 & 7;
        float v[8];
        ld8f(Sg + (size_t)r * DV + c16 * 8, v);
        st_chunk(sm + OFF_S, (uint32_t)p * 16384 + swz(r, ch), v);
        ld8f(dSg + (size_t)r * DV + c16 * 8, v);
        st_chunk(sm + OFF_DS, (uint32_t)p * 16384 + swz(r, ch), v);
    }
    const float *Ug = a.w.Un + ci * C * DV, *Gg = a.w.G + ci * C * DK;
    const float gC = Gg[(size_t)(C - 1) * DK];
    for (int x = tid; x < C * 16; x += NTHREADS) {     // U, dO, Kbar: 64 rows x 16 chunks
        const int r = x >> 4, c16 = x & 15, p = c16 >> 3, ch = c16 & 7;
        const uint32_t o = (uint32_t)p * 8192 + swz(r, ch);
        float v[8];
        ld8f(Ug + (size_t)r * DV + c16 * 8, v);
        st_chunk(sm + OFF_U, o, v);
        const size_t row = ((size_t)b * T + t0 + r) * H + h;
        if (r < L) {
            ld8h(reinterpret_cast<const __nv_bfloat16 *>(a.dout) + row * DV + c16 * 8, v);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = 0.f;
        }
        st_chunk(sm + OFF_DO, o, v);
        if (r < L) {
            ld8h(reinterpret_cast<const __nv_bfloat16 *>(a.k) + row * DK + c16 * 8, v);
            const float f = __expf(gC - Gg[(size_t)r * DK]);
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] *= f;
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = 0.f;
        }
        st_chunk(sm + OFF_KB, o, v);
    }
    const float *Pg = a.w.P + ci * C * C;
    for (int x = tid; x < C * 8; x += NTHREADS) {      // P: 64 rows x 8 chunks
        const int r = x >> 3, ch = x & 7;
        float v[8];
        ld8f(Pg + (size_t)r * C + ch * 8, v);
        st_chunk(sm + OFF_P, swz(r, ch), v);
    }
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tl = tbase + ((uint32_t)(warp * 32) << 16);
    const int row = warp * 32 + lane;  // TMEM lane owned by this thread

    // ---- dU^T, Qd^T, Tm^T ----
    if (tid == 0) {
        const uint32_t sS = smem_u32(sm + OFF_S), sD = smem_u32(sm + OFF_DS), sU = smem_u32(sm + OFF_U);
        const uint32_t sO = smem_u32(sm + OFF_DO), sK = smem_u32(sm + OFF_KB), sP = smem_u32(sm + OFF_P);
        const uint32_t id_a1 = idesc_bf16(128, 64, 1, 1), id_a2 = idesc_bf16(128, 64, 1, 0);
        const uint32_t id_kk = idesc_bf16(128, 64, 0, 0);
#pragma unroll
        for (int st = 0; st < 4; ++st)  // dO^T P
            mma_bf16(tbase + TM_DUT, sdesc(sO + st * 2048, 8192, 1024), sdesc(sP + st * 2048, 1024, 1024), id_a1,
                     st > 0);
#pragma unroll
        for (int st = 0; st < 8; ++st)  // + dS+^T Kbar^T
            mma_bf16(tbase + TM_DUT, sdesc(sD + st * 2048, 16384, 1024),
                     sdesc(sK + (st >> 2) * 8192 + (st & 3) * 32, 16, 1024), id_a2, 1);
#pragma unroll
        for (int st = 0; st < 8; ++st)  // Qd^T = S dO^T
            mma_bf16(tbase + TM_QD, sdesc(sS + (st >> 2) * 16384 + (st & 3) * 32, 16, 1024),
                     sdesc(sO + (st >> 2) * 8192 + (st & 3) * 32, 16, 1024), id_kk, st > 0);
#pragma unroll
        for (int st = 0; st < 8; ++st)  // Tm^T = dS+ U^T
            mma_bf16(tbase + TM_TM, sdesc(sD + (st >> 2) * 16384 + (st & 3) * 32, 16, 1024),
                     sdesc(sU + (st >> 2) * 8192 + (st & 3) * 32, 16, 1024), id_kk, st > 0);
        mma_commit(bar);
    }
    mbar_wait(bar, 0, abort_flag);
    fence_after_sync();
    const bool ok1 = !named_sync_any(1, NTHREADS, *abort_flag != 0);
    if (ok1) {
        float v[64];
        // dU (thread = value column j)
        tmem_row64(tl + TM_DUT, v);
        const int j = row;
        for (int r = 0; r < C; ++r) {
            float x = v[r];
            if (a.du && r < L)
                x += __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(a.du)[(((size_t)b * T + t0 + r) * H + h) * DV + j]);
            v[r] = x;
            a.w.dUn[(ci * C + r) * DV + j] = x;
        }
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) st_chunk(sm + OFF_DUT, swz(j, ch), v + ch * 8);
        // Qd, Tm (thread = key channel c)
        const int c = row;
        tmem_row64(tl + TM_QD, v);
        for (int r = 0; r < C; ++r) a.w.Qd[(ci * C + r) * DK + c] = v[r];
        tmem_row64(tl + TM_TM, v);
        for (int r = 0; r < C; ++r) a.w.Tm[(ci * C + r) * DK + c] = v[r];
        // RS[c] = sum_j S[c][j] dS+[c][j]
        float rs = 0.f;
        const float4 *s4 = reinterpret_cast<const float4 *>(Sg + (size_t)c * DV);
        const float4 *d4 = reinterpret_cast<const float4 *>(dSg + (size_t)c * DV);
        for (int q = 0; q < DV / 4; ++q) {
            const float4 x = s4[q], y = d4[q];
            rs += x.x * y.x + x.y * y.y + x.z * y.z + x.w * y.w;
        }
        a.w.RS[ci * DK + c] = rs;
    }
    fence_proxy_async();
    fence_before_sync();
    const bool ok2 = ok1 && !named_sync_any(1, NTHREADS, *abort_flag != 0);
    // ---- dWm^T = -S dU^T ----
    if (ok2) {
        if (tid == 0) {
            fence_after_sync();
            const uint32_t sS = smem_u32(sm + OFF_S), sT = smem_u32(sm + OFF_DUT);
            const uint32_t id = idesc_bf16(128, 64, 0, 1, 1);
#pragma unroll
            for (int st = 0; st < 8; ++st)
                mma_bf16(tbase + TM_DW, sdesc(sS + (st >> 2) * 16384 + (st & 3) * 32, 16, 1024),
                         sdesc(sT + st * 2048, 1024, 1024), id, st > 0);
            mma_commit(bar);
        }
        mbar_wait(bar, 1, abort_flag);
        fence_after_sync();
        if (!named_sync_any(1, NTHREADS, *abort_flag != 0)) {
            float v[64];
            tmem_row64(tl + TM_DW, v);
            for (int r = 0; r < C; ++r) a.w.dWm[(ci * C + r) * DK + row] = v[r];
        }
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == 0) tmem_dealloc(tbase, TM_COLS);
}

}  // namespace tcb

cudaError_t tc_bwd_state(const Geo &g, const Tensors &t, const SimtWs &w, cudaStream_t s, Rec &rec) {
    using namespace tcb;
    Args a;
    a.k = t.k; a.dout = t.dout; a.du = t.du; a.w = w;
    a.B = g.B; a.T = g.T; a.H = g.H; a.N = g.N;
    const size_t smem = SMEM_BYTES + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_bwd_state_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    rec.mark(s);
    k_bwd_state_tc<<<dim3(g.N, g.H, g.B), NTHREADS, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace dr
