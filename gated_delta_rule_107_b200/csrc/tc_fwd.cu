// tc_fwd.cu -- fused chunkwise forward on 5th-generation tensor cores (sm_100a).
//
// One CTA per (batch b, head h, half of the value dimension): it walks the
// chunks of 64 tokens in order, carrying its 128 x 64 slice of the fp32 state
// S in registers, and does every step of the chunked recurrence of
// "线性注意力架构演进与Kimi Delta Attention创新实践" (sections 2.1, 6.1, 6.2, 7.1)
// on chip: no intermediate touches HBM.  Per chunk, with g the in-chunk
// cumulative log gate, every matrix product is one tcgen05 MMA with M = 128,
// obtained by stacking two 64-row operands:
//
//   P1   [beta k ; q] . k^T          -> A (rows 0-63), P (rows 64-127)
//        (the scalar gate factor e^{g_r - g_i} <= 1 is applied exactly in the
//         epilogue)
//   T  = (I + A)^-1                    blocked forward substitution (CUDA cores)
//   IPT  R = [I ; P] . T  = [T ; P T]
//   P3   X = R . (beta e^{g} k)       -> [W ; P W]
//   P4   D = R . (beta v)             -> [U~ ; P U~]   (initial accumulator)
//        A_chain = [-W ; e^{g} q - P W]
//   C1   D += A_chain . S             -> rows 0-63: U = U~ - W S (write values u)
//                                        rows 64-127: O = Qtil S + P U
//   C3   E = Kbar^T . U                (Kbar = k e^{g_C - g})
//        S <- Diag(e^{g_C}) S + E      (fp32, registers)
//
// Serves Gated DeltaNet and DeltaNet (KDA's channel-wise gates take the split
// path at dv = 128 and the CUDA-core path otherwise).
//
// Warp roles: warp 0 = producer (TMA loads of q, k, v; plain loads of the
// scalar gate and beta); warps 1-4 = one warpgroup
// that does all epilogues / CUDA-core work and issues the MMAs from one elected
// thread.  Every wait is bounded (about 1 s); on expiry the kernel raises the
// device error word and leaves through the common teardown (TMEM freed).
#include "tc_host.cuh"
#include "tc_path.cuh"
#include "tc_ptx.cuh"
#include "tc_tile.cuh"

namespace dr {
namespace tcf {

using namespace dr::tc;

constexpr int C = 64;      // chunk length
constexpr int DK = 128;    // key dimension
constexpr int DVB = 64;    // state columns per CTA
constexpr int NTHREADS = 160;

// ---- shared memory map (bytes from a 1024-aligned base) ----
constexpr uint32_t SLOT = 32768;               // input slot: q (2 panels) + k (2 panels)
constexpr uint32_t IN_Q = 0, IN_K = 16384;
constexpr uint32_t OFF_V = 2 * SLOT;           //  8K  v (64 tokens x 64), scaled in place to beta v
constexpr uint32_t OFF_PA = OFF_V + 8192;      // 32K  [beta k ; q] : panel p at +16K p, 128 rows
constexpr uint32_t OFF_BKT = OFF_PA + 32768;   // 16K  beta e^{g} k (token rows, 2 panels of 8K)
constexpr uint32_t OFF_KB = OFF_BKT + 16384;   // 16K  Kbar (token rows, 2 panels of 8K)
constexpr uint32_t OFF_IPR = OFF_KB + 16384;   // 16K  [I ; P] then R (128 rows, 1 panel)
constexpr uint32_t OFF_T = OFF_IPR + 16384;    //  8K  T (64 rows, 1 panel), MN-major B
constexpr uint32_t OFF_AC = OFF_T + 8192;      // 32K  A_chain (128 rows, 2 panels of 16K); scratch in M3
constexpr uint32_t OFF_U = OFF_AC + 32768;     //  8K  U (64 token rows, 1 panel)
constexpr uint32_t OFF_S = OFF_U + 8192;       // 16K  bf16 S (128 rows, 1 panel)
constexpr uint32_t OFF_MISC = OFF_S + 16384;   //  4K  barriers and small vectors
constexpr uint32_t SMEM_BYTES = OFF_MISC + 4096;

// misc sub-offsets
constexpr uint32_t M_BAR = 0;      // 8 mbarriers
constexpr uint32_t M_TMEM = 64;    // TMEM base address
constexpr uint32_t M_ABORT = 68;   // abort flag
constexpr uint32_t M_GB = 128;     // [2 slots][2][64] floats: raw log gate, beta
constexpr uint32_t M_GC = M_GB + 1024;    // [64] cumulative g (Gated)
constexpr uint32_t M_FAC = M_GC + 256;    // [4][64] row factors: beta, beta e^g, e^{gC-g}, e^g
constexpr uint32_t M_GAM = M_FAC + 1024;  // [128] e^{g_C} per channel
static_assert(M_GAM + 512 <= 4096, "misc overflow");

// TMEM columns
constexpr uint32_t TM_G1 = 0;    // 64: P1 output, then R
constexpr uint32_t TM_X = 64;    // 128: P3 output
constexpr uint32_t TM_D = 192;   // 64: chain accumulator
constexpr uint32_t TM_E = 256;   // 64: C3 output
constexpr uint32_t TM_COLS = 512;

// barrier indices
enum { B_FULL0 = 0, B_FULL1, B_EMPTY0, B_EMPTY1, B_VFULL, B_VEMPTY, B_MMA, B_NUM };

struct Args {
    const void *alpha;   // raw log gate (Gated: [B,T,H])
    const void *beta;    // [B,T,H]
    const float *S0;     // [B,H,dk,dv] or null
    void *out, *u;       // [B,T,H,dv]
    float *ST;           // [B,H,dk,dv] or null
    int B, T, H, dv, N;
};

template <int VAR>
__global__ void __launch_bounds__(NTHREADS, 1)
    k_fwd_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_v, Args a) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    static_assert(VAR != VAR_KDA, "channel-wise gates take the split or the CUDA-core path");
    constexpr int NSLOT = 2;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + OFF_MISC + M_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC + M_TMEM);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + OFF_MISC + M_ABORT);
    float *gb = reinterpret_cast<float *>(sm + OFF_MISC + M_GB);      // [slot][0: loga, 1: beta][64]
    float *gc = reinterpret_cast<float *>(sm + OFF_MISC + M_GC);
    float *fac = reinterpret_cast<float *>(sm + OFF_MISC + M_FAC);    // [4][64]
    float *gam = reinterpret_cast<float *>(sm + OFF_MISC + M_GAM);

    const int half = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int j0 = half * DVB;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = a.T, H = a.H, DV = a.dv, N = a.N;

    if (threadIdx.x == 0) {
        mbar_init(&bar[B_FULL0], 2);
        mbar_init(&bar[B_FULL1], 2);
        mbar_init(&bar[B_EMPTY0], 1);
        mbar_init(&bar[B_EMPTY1], 1);
        mbar_init(&bar[B_VFULL], 1);
        mbar_init(&bar[B_VEMPTY], 1);
        mbar_init(&bar[B_MMA], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, TM_COLS);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = *tmem_slot;

    if (warp == 0) {
        // ============================== producer ==============================
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
        }
        int issued[2] = {0, 0}, v_issued = 0;
        for (int m = 0; m < N; ++m) {
            const int s = m % NSLOT, use = m / NSLOT, t0 = m * C;
            bool ok = true;
            if (use > 0) ok = mbar_wait(&bar[B_EMPTY0 + s], (use - 1) & 1, abort_flag);
            if (!ok) break;
            unsigned char *slot = sm + s * SLOT;
            if (lane == 0) {
                const uint32_t bytes = 2 * 16384;
                mbar_arrive_tx(&bar[B_FULL0 + s], bytes);
                tma_load_4d(slot + IN_Q, &tm_q, 0, h, t0, b, &bar[B_FULL0 + s]);
                tma_load_4d(slot + IN_Q + 8192, &tm_q, 64, h, t0, b, &bar[B_FULL0 + s]);
                tma_load_4d(slot + IN_K, &tm_k, 0, h, t0, b, &bar[B_FULL0 + s]);
                tma_load_4d(slot + IN_K + 8192, &tm_k, 64, h, t0, b, &bar[B_FULL0 + s]);
            }
            float *gbs = gb + s * 128;
            for (int r = lane; r < C; r += 32) {
                const int t = t0 + r;
                const size_t row = ((size_t)b * T + t) * H + h;
                float lg = 0.f, bt = 0.f;
                if (t < T) {
                    if (VAR == VAR_GATED) lg = bf(a.alpha, row);
                    bt = bf(a.beta, row);
                }
                gbs[r] = lg;
                gbs[64 + r] = bt;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[B_FULL0 + s]);
            issued[s]++;
            // v: one buffer, released after the P4 MMA of the previous chunk
            if (m > 0 && !mbar_wait(&bar[B_VEMPTY], (m - 1) & 1, abort_flag)) break;
            if (lane == 0) {
                mbar_arrive_tx(&bar[B_VFULL], 8192);
                tma_load_4d(sm + OFF_V, &tm_v, j0, h, t0, b, &bar[B_VFULL]);
            }
            v_issued++;
        }
        if (*abort_flag) {
            // let issued copies land before the CTA retires (bounded)
            volatile int dummy = 0;
            for (int s = 0; s < NSLOT; ++s)
                if (issued[s] > 0) mbar_wait(&bar[B_FULL0 + s], (issued[s] - 1) & 1, &dummy, 100000000ull);
            if (v_issued > 0) mbar_wait(&bar[B_VFULL], (v_issued - 1) & 1, &dummy, 100000000ull);
        }
    } else {
        // ============================== math warpgroup ==============================
        const int wt = threadIdx.x - 32;                 // 0..127
        const int q4 = warp & 3;                         // TMEM lane quarter of this warp
        const int trow = q4 * 32 + lane;                 // TMEM lane / matrix row owned by this thread
        const uint32_t tl = tbase + ((uint32_t)(q4 * 32) << 16);  // this warp's lane base
        const bool elected = (wt == 0);
        uint32_t mma_phase = 0;
        bool mma_pending = false;

        auto wg_sync = [&]() { named_sync(1, 128); };
        // barrier over the warpgroup that also agrees on whether to abort
        auto wg_abort = [&]() -> bool { return named_sync_any(1, 128, *abort_flag != 0); };
        // Wait for the MMA commit; every thread then agrees on success.
        auto mma_wait = [&]() -> bool {
            mbar_wait(&bar[B_MMA], mma_phase & 1, abort_flag);
            mma_phase++;
            fence_after_sync();
            const bool ok = !wg_abort();
            if (ok) mma_pending = false;
            return ok;
        };
        auto issue_begin = [&]() { fence_after_sync(); };

        // state slice: thread trow owns S[trow][j0 .. j0+63]
        float S[DVB];
        {
            const float *s0 = a.S0 ? a.S0 + (((size_t)b * H + h) * DK + trow) * DV + j0 : nullptr;
#pragma unroll
            for (int j = 0; j < DVB; ++j) S[j] = s0 ? s0[j] : 0.f;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) st_chunk(sm + OFF_S, swz(trow, ch), S + ch * 8);
        }
        fence_proxy_async();
        wg_sync();

        for (int m = 0; m < N; ++m) {
            const int s = m % NSLOT, use = m / NSLOT, t0 = m * C;
            const int L = min(C, T - t0);
            unsigned char *slot = sm + s * SLOT;
            mbar_wait(&bar[B_FULL0 + s], use & 1, abort_flag);
            if (wg_abort()) break;
            const float *lg = gb + s * 128, *bt = gb + s * 128 + 64;
            // ------------------------------ M1: gates and operand tiles ------------------------------
            if (wt < 32) {
                // inclusive scan of the 64 log gates (two per lane)
                float x0 = lg[lane], x1 = lg[lane + 32];
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y0 = __shfl_up_sync(0xffffffffu, x0, o);
                    const float y1 = __shfl_up_sync(0xffffffffu, x1, o);
                    if (lane >= o) { x0 += y0; x1 += y1; }
                }
                x1 += __shfl_sync(0xffffffffu, x0, 31);
                const float gC = __shfl_sync(0xffffffffu, x1, 31);
                gc[lane] = x0;
                gc[lane + 32] = x1;
                fac[0 * 64 + lane] = bt[lane];
                fac[0 * 64 + lane + 32] = bt[lane + 32];
                fac[1 * 64 + lane] = bt[lane] * __expf(x0);
                fac[1 * 64 + lane + 32] = bt[lane + 32] * __expf(x1);
                fac[2 * 64 + lane] = __expf(gC - x0);
                fac[2 * 64 + lane + 32] = __expf(gC - x1);
                fac[3 * 64 + lane] = __expf(x0);
                fac[3 * 64 + lane + 32] = __expf(x1);
                const float eg = __expf(gC);
                for (int c = lane; c < DK; c += 32) gam[c] = eg;
            }
            wg_sync();
            // q, k -> [beta k ; q], beta e^g k, Kbar ; 64 rows x 16 chunks
            for (int x = wt; x < C * 16; x += 128) {
                const int r = x >> 4, j = x & 15, p = j >> 3;
                const uint32_t o = (uint32_t)p * 8192 + swz(r, j & 7);
                float kv[8], qv[8], w[8];
                ld_chunk(slot + IN_K, o, kv);
                ld_chunk(slot + IN_Q, o, qv);
                const float f0 = fac[r], f1 = fac[64 + r], f2 = fac[128 + r];
#pragma unroll
                for (int e = 0; e < 8; ++e) w[e] = f0 * kv[e];
                st_chunk(sm + OFF_PA, (uint32_t)p * 16384 + swz(r, j & 7), w);
                st_chunk(sm + OFF_PA, (uint32_t)p * 16384 + 8192 + swz(r, j & 7), qv);
#pragma unroll
                for (int e = 0; e < 8; ++e) w[e] = f1 * kv[e];
                st_chunk(sm + OFF_BKT, o, w);
#pragma unroll
                for (int e = 0; e < 8; ++e) w[e] = f2 * kv[e];
                st_chunk(sm + OFF_KB, o, w);
            }
            fence_proxy_async();
            wg_sync();
            // ------------------------------ P1 ------------------------------
            if (elected) {
                issue_begin();
                const uint32_t idesc = idesc_bf16(128, 64, 0, 0);
                const uint32_t pa = smem_u32(sm + OFF_PA), kt = smem_u32(slot + IN_K);
#pragma unroll
                for (int st = 0; st < 8; ++st)
                    mma_bf16(tbase + TM_G1, sdesc(pa + (st >> 2) * 16384 + (st & 3) * 32, 16, 1024),
                             sdesc(kt + (st >> 2) * 8192 + (st & 3) * 32, 16, 1024), idesc, st > 0);
                mma_commit(&bar[B_MMA]);
            }
            mma_pending = true;
            if (!mma_wait()) break;
            // ------------------------------ M3: A, P, inverse ------------------------------
            {
                float g1[64];
                tmem_row64(tl + TM_G1, g1);
                float *Asc = reinterpret_cast<float *>(sm + OFF_AC);       // [64][65]
                if (trow < 64) {
                    const int r = trow;
                    const float gr = (VAR == VAR_GATED) ? gc[r] : 0.f;
#pragma unroll
                    for (int i = 0; i < 64; ++i) {
                        float v = (i < r) ? g1[i] : 0.f;
                        if (VAR == VAR_GATED && i < r) v *= __expf(gr - gc[i]);
                        Asc[r * 65 + i] = v;
                    }
                    // identity row of [I ; P]
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        float w[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) w[e] = (ch * 8 + e == r) ? 1.f : 0.f;
                        st_chunk(sm + OFF_IPR, swz(r, ch), w);
                    }
                } else {
                    const int r = trow - 64;
                    const float gr = (VAR == VAR_GATED) ? gc[r] : 0.f;
#pragma unroll
                    for (int i = 0; i < 64; ++i) {
                        float v = (i <= r) ? g1[i] : 0.f;
                        if (VAR == VAR_GATED && i <= r) v *= __expf(gr - gc[i]);
                        g1[i] = v;
                    }
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) st_chunk(sm + OFF_IPR, swz(trow, ch), g1 + ch * 8);
                }
                fence_before_sync();
                wg_sync();
                // blocked inverse of the unit lower-triangular I + A, fp32, into Tf [64][65]
                float *Tf = reinterpret_cast<float *>(slot);                // the input slot is free after P1
                float *Ys = reinterpret_cast<float *>(sm + OFF_AC + 64 * 65 * 4);  // [3][16][17]
                {
                    const int R = wt >> 5, j = lane;
                    if (j < 16) {
                        float t[16];
#pragma unroll
                        for (int r = 0; r < 16; ++r) {
                            float acc = (r == j) ? 1.f : 0.f;
#pragma unroll
                            for (int i = 0; i < r; ++i) acc -= Asc[(16 * R + r) * 65 + 16 * R + i] * t[i];
                            t[r] = acc;
                        }
#pragma unroll
                        for (int r = 0; r < 16; ++r) Tf[(16 * R + r) * 65 + 16 * R + j] = t[r];
                    }
                }
                wg_sync();
                for (int d = 1; d < 4; ++d) {
                    const int nb = 4 - d;
                    for (int e = wt; e < nb * 256; e += 128) {
                        const int I = e >> 8, y = (e >> 4) & 15, x = e & 15, R = I + d;
                        float acc = 0.f;
                        for (int J = I; J < R; ++J)
#pragma unroll
                            for (int k = 0; k < 16; ++k)
                                acc += Asc[(16 * R + y) * 65 + 16 * J + k] * Tf[(16 * J + k) * 65 + 16 * I + x];
                        Ys[(I * 16 + y) * 17 + x] = acc;
                    }
                    wg_sync();
                    for (int e = wt; e < nb * 256; e += 128) {
                        const int I = e >> 8, y = (e >> 4) & 15, x = e & 15, R = I + d;
                        float acc = 0.f;
                        for (int k = 0; k <= y; ++k) acc += Tf[(16 * R + y) * 65 + 16 * R + k] * Ys[(I * 16 + k) * 17 + x];
                        Tf[(16 * R + y) * 65 + 16 * I + x] = -acc;
                    }
                    wg_sync();
                }
                // T (row-major, bf16) -> MN-major B tile
                if (wt < 64) {
                    const int i = wt;
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        float w[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int n = ch * 8 + e;
                            w[e] = (n <= i) ? Tf[i * 65 + n] : 0.f;
                        }
                        st_chunk(sm + OFF_T, swz(i, ch), w);
                    }
                }
                fence_proxy_async();
                wg_sync();
                if (wt == 0) mbar_arrive(&bar[B_EMPTY0 + s]);   // q / k slot (and scratch) free
            }
            // ------------------------------ IPT: R = [I;P] T ------------------------------
            if (elected) {
                issue_begin();
                const uint32_t idesc = idesc_bf16(128, 64, 0, 1);
                const uint32_t ip = smem_u32(sm + OFF_IPR), tt = smem_u32(sm + OFF_T);
#pragma unroll
                for (int st = 0; st < 4; ++st)
                    mma_bf16(tbase + TM_G1, sdesc(ip + st * 32, 16, 1024), sdesc(tt + st * 2048, 1024, 1024), idesc,
                             st > 0);
                mma_commit(&bar[B_MMA]);
            }
            mma_pending = true;
            if (!mma_wait()) break;
            // ------------------------------ M5: R -> bf16 ------------------------------
            {
                float rv[64];
                tmem_row64(tl + TM_G1, rv);
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) st_chunk(sm + OFF_IPR, swz(trow, ch), rv + ch * 8);
                // beta v in place (64 rows x 8 chunks)
                mbar_wait(&bar[B_VFULL], m & 1, abort_flag);
                fence_before_sync();
                if (wg_abort()) break;
                for (int x = wt; x < C * 8; x += 128) {
                    const int r = x >> 3, ch = x & 7;
                    float vv[8];
                    ld_chunk(sm + OFF_V, swz(r, ch), vv);
                    const float f = fac[r];
#pragma unroll
                    for (int e = 0; e < 8; ++e) vv[e] *= f;
                    st_chunk(sm + OFF_V, swz(r, ch), vv);
                }
                fence_proxy_async();
                wg_sync();
            }
            // ------------------------------ P3, P4 ------------------------------
            if (elected) {
                issue_begin();
                const uint32_t r0 = smem_u32(sm + OFF_IPR), bk = smem_u32(sm + OFF_BKT), vv = smem_u32(sm + OFF_V);
                const uint32_t id3 = idesc_bf16(128, 128, 0, 1), id4 = idesc_bf16(128, 64, 0, 1);
#pragma unroll
                for (int st = 0; st < 4; ++st)
                    mma_bf16(tbase + TM_X, sdesc(r0 + st * 32, 16, 1024), sdesc(bk + st * 2048, 8192, 1024), id3,
                             st > 0);
#pragma unroll
                for (int st = 0; st < 4; ++st)
                    mma_bf16(tbase + TM_D, sdesc(r0 + st * 32, 16, 1024), sdesc(vv + st * 2048, 1024, 1024), id4,
                             st > 0);
                mma_commit(&bar[B_MMA]);
            }
            mma_pending = true;
            if (!mma_wait()) break;
            if (wt == 0) mbar_arrive(&bar[B_VEMPTY]);
            // ------------------------------ M7: A_chain ------------------------------
            {
                const int r = trow;
#pragma unroll
                for (int half2 = 0; half2 < 2; ++half2) {
                    float xv[64];
                    tmem_row64(tl + TM_X + half2 * 64, xv);
                    if (r < 64) {
#pragma unroll
                        for (int i = 0; i < 64; ++i) xv[i] = -xv[i];
                    } else {
                        const int rr = r - 64;
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch) {
                            float qv[8];
                            ld_chunk(sm + OFF_PA, (uint32_t)half2 * 16384 + 8192 + swz(rr, ch), qv);
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const float sc = fac[192 + rr];
                                xv[ch * 8 + e] = qv[e] * sc - xv[ch * 8 + e];
                            }
                        }
                    }
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) st_chunk(sm + OFF_AC, (uint32_t)half2 * 16384 + swz(r, ch), xv + ch * 8);
                }
                fence_before_sync();
                fence_proxy_async();
                wg_sync();
            }
            // ------------------------------ C1: D += A_chain . S ------------------------------
            if (elected) {
                issue_begin();
                const uint32_t ac = smem_u32(sm + OFF_AC), ss = smem_u32(sm + OFF_S);
                const uint32_t idesc = idesc_bf16(128, 64, 0, 1);
#pragma unroll
                for (int st = 0; st < 8; ++st)
                    mma_bf16(tbase + TM_D, sdesc(ac + (st >> 2) * 16384 + (st & 3) * 32, 16, 1024),
                             sdesc(ss + st * 2048, 1024, 1024), idesc, 1);
                mma_commit(&bar[B_MMA]);
            }
            mma_pending = true;
            if (!mma_wait()) break;
            // ------------------------------ C2: U and O ------------------------------
            {
                float dv[64];
                tmem_row64(tl + TM_D, dv);
                if (trow < 64) {
                    const int r = trow;
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) st_chunk(sm + OFF_U, swz(r, ch), dv + ch * 8);
                    if (a.u && r < L) {
                        uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(a.u) +
                                                               (((size_t)b * T + t0 + r) * H + h) * DV + j0);
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch) {
                            uint4 w;
                            w.x = pack_bf16(dv[ch * 8 + 0], dv[ch * 8 + 1]);
                            w.y = pack_bf16(dv[ch * 8 + 2], dv[ch * 8 + 3]);
                            w.z = pack_bf16(dv[ch * 8 + 4], dv[ch * 8 + 5]);
                            w.w = pack_bf16(dv[ch * 8 + 6], dv[ch * 8 + 7]);
                            dst[ch] = w;
                        }
                    }
                } else {
                    const int r = trow - 64;
                    if (r < L) {
                        uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<__nv_bfloat16 *>(a.out) +
                                                               (((size_t)b * T + t0 + r) * H + h) * DV + j0);
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch) {
                            uint4 w;
                            w.x = pack_bf16(dv[ch * 8 + 0], dv[ch * 8 + 1]);
                            w.y = pack_bf16(dv[ch * 8 + 2], dv[ch * 8 + 3]);
                            w.z = pack_bf16(dv[ch * 8 + 4], dv[ch * 8 + 5]);
                            w.w = pack_bf16(dv[ch * 8 + 6], dv[ch * 8 + 7]);
                            dst[ch] = w;
                        }
                    }
                }
                fence_before_sync();
                fence_proxy_async();
                wg_sync();
            }
            // ------------------------------ C3: E = Kbar^T U ------------------------------
            if (elected) {
                issue_begin();
                const uint32_t kb = smem_u32(sm + OFF_KB), uu = smem_u32(sm + OFF_U);
                const uint32_t idesc = idesc_bf16(128, 64, 1, 1);
#pragma unroll
                for (int st = 0; st < 4; ++st)
                    mma_bf16(tbase + TM_E, sdesc(kb + st * 2048, 8192, 1024), sdesc(uu + st * 2048, 1024, 1024), idesc,
                             st > 0);
                mma_commit(&bar[B_MMA]);
            }
            mma_pending = true;
            if (!mma_wait()) break;
            // ------------------------------ C4: S <- gamma S + E ------------------------------
            {
                float ev[64];
                tmem_row64(tl + TM_E, ev);
                const float gmc = gam[trow];
#pragma unroll
                for (int j = 0; j < DVB; ++j) S[j] = gmc * S[j] + ev[j];
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) st_chunk(sm + OFF_S, swz(trow, ch), S + ch * 8);
                fence_before_sync();
                fence_proxy_async();
                wg_sync();
            }
        }
        if (*abort_flag == 0) {
            if (a.ST) {
                float *dst = a.ST + (((size_t)b * H + h) * DK + trow) * DV + j0;
#pragma unroll
                for (int j = 0; j < DVB; j += 4)
                    *reinterpret_cast<float4 *>(dst + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
            }
        } else if (mma_pending) {
            volatile int dummy = 0;
            mbar_wait(&bar[B_MMA], mma_phase & 1, &dummy, 100000000ull);
        }
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == 0) tmem_dealloc(tbase, TM_COLS);
}

}  // namespace tcf

bool tc_fwd_supported(const Geo &g, bool bf16) {
    return bf16 && g.C == tcf::C && g.dk == tcf::DK && (g.dv == 64 || g.dv == 128) && g.variant != VAR_KDA;
}

int tc_fwd_launches(const Geo &g, const char **names, int max_names) {
    (void)g;
    if (names && max_names > 0) names[0] = "k_fwd_tc";
    return 1;
}

cudaError_t tc_fwd(const Geo &g, const Tensors &t, void *workspace, cudaStream_t s, Rec &rec) {
    using namespace tcf;

    CUtensorMap mq, mk, mv;
    const uint64_t Bn = g.B, T = g.T, H = g.H;
    bool ok = tc::make_map_4d_bf16(&mq, t.q, DK, H, T, Bn, 64) && tc::make_map_4d_bf16(&mk, t.k, DK, H, T, Bn, 64) &&
              tc::make_map_4d_bf16(&mv, t.v, g.dv, H, T, Bn, 64);
    if (!ok || g.variant == VAR_KDA) return cudaErrorInvalidValue;
    Args a;
    a.alpha = t.alpha; a.beta = t.beta; a.S0 = t.S0; a.out = t.out; a.u = t.u; a.ST = t.S_T;
    a.B = g.B; a.T = g.T; a.H = g.H; a.dv = g.dv; a.N = g.N;
    const dim3 grid(g.dv / DVB, g.H, g.B);
    const size_t smem = SMEM_BYTES + 1024;
    cudaError_t e;
    switch (g.variant) {
        case VAR_DELTANET:
            e = cudaFuncSetAttribute(k_fwd_tc<VAR_DELTANET>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
            rec.mark(s);
            k_fwd_tc<VAR_DELTANET><<<grid, NTHREADS, smem, s>>>(mq, mk, mv, a);
            break;
        case VAR_GATED:
            e = cudaFuncSetAttribute(k_fwd_tc<VAR_GATED>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
            rec.mark(s);
            k_fwd_tc<VAR_GATED><<<grid, NTHREADS, smem, s>>>(mq, mk, mv, a);
            break;
        default:
            return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace dr
