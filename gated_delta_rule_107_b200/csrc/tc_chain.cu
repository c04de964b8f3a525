// tc_chain.cu -- the serial state chains of the chunked gated delta rule on tcgen05
// (Gated DeltaNet and DeltaNet; bf16 I/O, dk = dv = 128, C = 64).
//
// Chunked form of "线性注意力架构演进与Kimi Delta Attention创新实践" (sections 2.1, 6.1,
// 6.2, 7.1), given the per-chunk products of tc_prep.cu (W, U~, P, g).  One CTA per (b, h, 64 value channels) walks the chunks in order; the state
// block (128 key rows x 64 value columns) stays in fp32 registers, one row per thread, with a
// bf16 copy in shared memory as the MMA operand.
//
// Forward chain, chunk n, S = S_n:
//   D  = [W ; q] S                  rows 0-63: W S, rows 64-127: q S
//   U  = U~ - W S                   the write values (the forward's u)
//   O' = P U                        (M = 128 MMA; rows 0-63 discarded)
//   o  = diag(e^g) q S + O'
//   S_{n+1} = e^{g_C} S + k^T (e^{g_C - g} U)
// Reverse chain, chunk n from last to first, dS+ = dL/dS_{n+1}:
//   dU = du + P^T dO + diag(e^{g_C - g}) k dS+         (stored: the gradient kernel reads it)
//   dL/dS_n = e^{g_C} dS+ + q^T diag(e^g) dO - W^T dU
//   and the row sums U_r . (diag(e^{g_C - g}) k dS+)_r of its 64 columns (a term of d log alpha)
//
// Warp 0 is a TMA producer that keeps two chunks of operands in flight; warps 1-8 run the
// chain (a TMEM lane = a state row; two warps per lane quarter split the value columns).
// Every wait is bounded (~1 s) and aborts are agreed on by the chain warps.
#include <limits.h>

#include "tc_host.cuh"
#include "tc_path.cuh"
#include "tc_ptx.cuh"
#include "tc_tile.cuh"

namespace dr {
namespace tch {

using namespace dr::tc;
using dr::tcf::ld_chunk;
using dr::tcf::st_chunk;
using dr::tcf::tmem_row64;

constexpr int C = 64, DK = 128, DV = 128, DVB = 64;
constexpr int NTHREADS = 288;  // warp 0 producer, warps 1-8 chain
// shared memory (bytes from a 1024-aligned base): two stages of 80K, then the chain's tiles
constexpr uint32_t STAGE = 81920;
// forward stage: [W_p0 | q_p0 | W_p1 | q_p1], [U~ (this CTA's 64 columns) | P], [k_p0 | k_p1],
// and for the fused forward the output gate logits (this CTA's 64 columns)
constexpr uint32_t FS_WQ = 0, FS_UP = 32768, FS_K = 49152, FS_G = 65536;
// reverse stage: k, q, W (2 panels each); dO (this CTA's 64 columns); P; du, U (this CTA's 64 columns)
constexpr uint32_t RS_K = 0, RS_Q = 16384, RS_W = 32768, RS_DO = 49152, RS_P = 57344, RS_DX = 65536,
                   RS_UN = 73728;
constexpr uint32_t OFF_S = 2 * STAGE;         // 16K  bf16 state [c][j]
constexpr uint32_t OFF_U = OFF_S + 16384;     //  8K  U [r][j]        (reverse: dU [r][j])
constexpr uint32_t OFF_UD = OFF_U + 8192;     //  8K  e^{g_C - g} U [r][j]
constexpr uint32_t OFF_O = OFF_UD + 8192;     //  8K  o [r][j] (staging of the TMA store)
constexpr uint32_t OFF_Y = OFF_O + 8192;      //  8K  fused forward: y [r][j] (staging)
constexpr uint32_t OFF_O1 = OFF_Y + 8192;     //  8K  fused forward: o of odd chunks (even: OFF_O)
constexpr uint32_t OFF_MISC = OFF_O1 + 8192;  //  4K
constexpr uint32_t SMEM_BYTES = OFF_MISC + 4096;
// misc
constexpr uint32_t M_BAR = 0;  // FULL0, FULL1, EMPTY0, EMPTY1, MMA
constexpr uint32_t M_TMEM = 128, M_ABORT = 132;
constexpr uint32_t M_CF = 256;  // per stage: [0..63] e^{g_C - g}, [64..127] e^g, [128] e^{g_C}
constexpr uint32_t M_SKP = M_CF + 2 * 132 * 4;  // reverse: [2 column halves][64] row-sum partials;
                                                // fused forward: the same for o's squares
constexpr uint32_t M_XS = M_SKP + 512;          // fused forward: [4 slots (chunk mod 4)][64] the partner's
                                                // row sums of squares (written by the partner CTA)
constexpr uint32_t M_WN = M_XS + 1024;          // fused forward: this CTA's 64 RMSNorm weights
constexpr uint32_t M_SQ1 = M_WN + 256;          // fused forward: o's row-sum partials of odd chunks
                                                // (even chunks: M_SKP)
// B_XS0..3 (fused forward): the partner's row sums of a chunk (mod 4) have arrived (256 bytes of
// asynchronous remote stores, armed by this CTA)
enum { B_FULL0 = 0, B_FULL1, B_EMPTY0, B_EMPTY1, B_MMA, B_XS0, B_XS1, B_XS2, B_XS3, B_NUM };
static_assert(B_NUM * 8 <= M_TMEM && M_SQ1 + 512 <= 4096 && M_WN % 16 == 0, "misc overflow");
constexpr float POST_EPS = 1e-6f;  // y = o / sqrt(mean(o^2) + eps) w sigmoid(gate)

struct FMaps {
    CUtensorMap q, k;       // [B, T, H, 128] bf16; box 64 x 64 tokens (KDA: the workspace's
                            // q e^g and k e^{g_C - g}, [chunks * 64][128], box 64 x 64)
    CUtensorMap W, Ut;      // [chunks * 64][128] bf16; box 64 x 64
    CUtensorMap P;          // [chunks * 64][64] bf16; box 64 x 64
    CUtensorMap out, u;     // forward outputs [B, T, H, 128] (stores)
    CUtensorMap Sn, Un;     // recompute outputs: [chunks * 128][128] box 64 x 128, [chunks * 64][128] (stores)
    CUtensorMap gate, y;    // fused forward: output gate logits (load) and y (store), [B, T, H, 128]
};
struct RMaps {
    CUtensorMap q, k, dout, du;  // [B, T, H, 128] bf16
    CUtensorMap W, Un;           // [chunks * 64][128] bf16 (loads)
    CUtensorMap P;               // [chunks * 64][64] bf16 (load)
    CUtensorMap dUn;             // [chunks * 64][128] bf16 (store)
    CUtensorMap dSn;             // [chunks * 128][128] bf16, box 64 x 128 (store)
};
struct Args {
    const float *gb;          // [chunks][2][64]: g, beta
    const float *S0;          // forward: S0; reverse: dS_T (fp32 [B, H, 128, 128], may be null)
    float *ST;                // forward: S_T; reverse: dS0 (may be null)
    int has_out, has_u;       // forward outputs requested
    float *skt;               // reverse output
    int B, T, H, N, has_du;
    const float *egc;         // KDA forward: [chunks][128] e^{g_C} per key channel
    const float *rn;          // fused forward: [chunks][2][64] 1 / |k_r|, 1 / |q_r|
    const float *wn;          // fused forward: RMSNorm weight [128]
    int m0, m1;               // the chunks [m0, m1) of each sequence (m1 = 0: to the end); forward: S0
                              // the state entering chunk m0, ST the state after chunk m1 - 1; reverse:
                              // S0 = dL/dS after chunk m1 - 1, ST = dL/dS entering chunk m0
};

// The producer's gate factors of a chunk (e^{g_C - g}, e^g, e^{g_C}; fused forward: with the raw
// rows' norms folded in, k's rows by 1 / |k_r|, o's by 1 / |q_r|; KDA: e^{g_C} per key channel).
// Their inputs are fetched into registers before the producer waits for a free stage, so that the
// global loads' latency overlaps the wait.
struct FactorIn {
    float x[4], r[4], gc;
};
template <bool KDA, bool FUSED>
__device__ __forceinline__ void factors_fetch(const Args &a, size_t ci, int lane, FactorIn &f) {
    if (KDA) {
#pragma unroll
        for (int k = 0; k < 4; ++k) f.x[k] = a.egc[ci * 128 + lane + 32 * k];
    } else {
        const float *gg = a.gb + ci * 2 * C;
        f.gc = gg[C - 1];
        f.x[0] = gg[lane];
        f.x[1] = gg[lane + 32];
        if (FUSED) {
            const float *rr = a.rn + ci * 2 * C;
            f.r[0] = rr[lane];
            f.r[1] = rr[lane + 32];
            f.r[2] = rr[C + lane];
            f.r[3] = rr[C + lane + 32];
        }
    }
}
template <bool KDA, bool FUSED>
__device__ __forceinline__ void factors_store(const FactorIn &f, float *cf, int lane) {
    if (KDA) {
#pragma unroll
        for (int k = 0; k < 4; ++k) cf[lane + 32 * k] = f.x[k];
    } else {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int r = lane + 32 * hh;
            cf[r] = __expf(f.gc - f.x[hh]) * (FUSED ? f.r[hh] : 1.f);
            cf[64 + r] = __expf(f.x[hh]) * (FUSED ? f.r[2 + hh] : 1.f);
        }
        if (lane == 0) cf[128] = __expf(f.gc);
    }
}

// sigmoid of a pair of bf16 values, as a pair of bf16: (1 + tanh(x / 2)) / 2 in packed bf16
// arithmetic (the hardware tanh approximation; x / 2 is exact)
__device__ __forceinline__ uint32_t sigmoid_bf16x2(uint32_t x) {
    constexpr uint32_t HALF2 = 0x3f003f00u;  // (0.5, 0.5)
    uint32_t hx, t, sg;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(hx) : "r"(x), "r"(HALF2));
    asm("tanh.approx.bf16x2 %0, %1;" : "=r"(t) : "r"(hx));
    asm("fma.rn.bf16x2 %0, %1, %2, %2;" : "=r"(sg) : "r"(t), "r"(HALF2));
    return sg;
}

// Chain thread layout: warps 1-8, two per TMEM lane quarter (warp & 3); the first four take
// value columns 0-31 of this CTA's 64, the other four columns 32-63.
struct ChainLane {
    int wc, q4, hf, trow, cb;
    __device__ ChainLane(int warp, int lane)
        : wc((warp - 1) * 32 + lane), q4(warp & 3), hf((warp - 1) >> 2), trow((warp & 3) * 32 + lane),
          cb(((warp - 1) >> 2) * 32) {}
};

// 32 fp32 columns of this thread's TMEM lane
__device__ __forceinline__ void tmem_row32(uint32_t taddr, float *v) {
    tmem_ld16(taddr, v);
    tmem_ld16(taddr + 16, v + 16);
    wait_ld();
}

// ====================================== forward chain ======================================
// MODE 0: forward (o, u, S_T); 1: recompute for the backward (S_n, U of every chunk);
// 2: forward that also keeps S_n and U for the backward; 3: the fused forward (raw q, k through
// the row norms; y = RMSNorm(o) w sigmoid(gate) in the output epilogue, the row sums of squares
// exchanged with the partner CTA of the cluster; o stored only when requested).
// KDA (MODE 0): q and k arrive gate-scaled (q e^g, k e^{g_C - g}), so the row factors are 1,
// and the state decays by row: S <- Diag(e^{g_C}) S + (k e^{g_C - g})^T U.
template <int MODE, int KDA>
__global__ void __launch_bounds__(NTHREADS, 1) k_chain_fwd(const __grid_constant__ FMaps mp, Args a) {
    constexpr bool OUT = MODE != 1, KEEP = MODE == 1 || MODE == 2, FUSED = MODE == 3;
    static_assert(!FUSED || !KDA, "the fused forward serves scalar gates");
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + OFF_MISC + M_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC + M_TMEM);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + OFF_MISC + M_ABORT);
    float *cf_all = reinterpret_cast<float *>(sm + OFF_MISC + M_CF);

    const int half = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int j0 = half * DVB;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = a.T, H = a.H, N = a.N;
    const int m0 = a.m0, NS = (a.m1 > 0 ? a.m1 : N) - m0;  // this launch's chunks: [m0, m0 + NS)
    const size_t ci0 = ((size_t)b * H + h) * N;

    if (threadIdx.x == 0) {
        for (int i = 0; i < B_NUM; ++i)
            mbar_init(&bar[i], (i == B_FULL0 || i == B_FULL1) ? 2 : 1);
        *abort_flag = 0;
        fence_mbar_init();
        if (FUSED)  // each exchange slot expects the partner's 64 row sums of chunks 0-3 (re-armed as consumed)
            for (int i = 0; i < 4; ++i) mbar_arrive_tx(&bar[B_XS0 + i], 64 * 4);
    }
    if (FUSED && threadIdx.x < DVB)
        reinterpret_cast<float *>(sm + OFF_MISC + M_WN)[threadIdx.x] = a.wn[j0 + threadIdx.x];
    if (warp == 0) tmem_alloc(tmem_slot, 512);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (FUSED) cluster_sync();  // the partner's barriers are initialised before any remote arrival
    const uint32_t tbase = *tmem_slot;

    if (warp == 0) {
        // ================================ producer ================================
        int issued[2] = {0, 0};
        FactorIn fin;
        for (int mi = 0; mi < NS; ++mi) {  // mi: this launch's chunk count so far (stages, phases)
            const int m = m0 + mi, s = mi & 1, t0 = m * C;
            const int ci = (int)(ci0 + m);
            factors_fetch<KDA != 0, FUSED>(a, (size_t)ci, lane, fin);
            if (mi >= 2 && !mbar_wait(&bar[B_EMPTY0 + s], ((mi >> 1) - 1) & 1, abort_flag)) break;
            unsigned char *st = sm + s * STAGE;
            if (lane == 0) {
                mbar_arrive_tx(&bar[B_FULL0 + s], (OUT ? 65536u : 40960u) + (FUSED ? 8192u : 0u));
                if (FUSED) tma_load_4d(st + FS_G, &mp.gate, j0, h, t0, b, &bar[B_FULL0 + s]);
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    tma_load_2d(st + FS_WQ + p * 16384, &mp.W, 64 * p, ci * C, &bar[B_FULL0 + s]);
                    if (KDA) {
                        if (OUT) tma_load_2d(st + FS_WQ + p * 16384 + 8192, &mp.q, 64 * p, ci * C, &bar[B_FULL0 + s]);
                        tma_load_2d(st + FS_K + p * 8192, &mp.k, 64 * p, ci * C, &bar[B_FULL0 + s]);
                    } else {
                        if (OUT) tma_load_4d(st + FS_WQ + p * 16384 + 8192, &mp.q, 64 * p, h, t0, b, &bar[B_FULL0 + s]);
                        tma_load_4d(st + FS_K + p * 8192, &mp.k, 64 * p, h, t0, b, &bar[B_FULL0 + s]);
                    }
                }
                tma_load_2d(st + FS_UP, &mp.Ut, j0, ci * C, &bar[B_FULL0 + s]);
                if (OUT) tma_load_2d(st + FS_UP + 8192, &mp.P, 0, ci * C, &bar[B_FULL0 + s]);
            }
            factors_store<KDA != 0, FUSED>(fin, cf_all + s * 132, lane);
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[B_FULL0 + s]);
            issued[s]++;
        }
        if (*abort_flag) {
            volatile int dummy = 0;
            for (int s = 0; s < 2; ++s)
                if (issued[s] > 0) mbar_wait(&bar[B_FULL0 + s], (issued[s] - 1) & 1, &dummy, 100000000ull);
        }
    } else {
        // ================================ chain ================================
        const ChainLane cl(warp, lane);
        const int wc = cl.wc, trow = cl.trow, hf = cl.hf, cb = cl.cb;
        const uint32_t tl = tbase + ((uint32_t)(cl.q4 * 32) << 16) + (uint32_t)cb;
        constexpr uint32_t TM_D = 0, TM_E = 256;  // D / O' double-buffered at 0 and 128
        const bool ostore = trow == 64 && hf == 0;  // issues the o stores
        uint32_t ph = 0;
        bool pending = false;
        auto wabort = [&](bool ok) -> bool { return named_sync_any(2, 256, !ok || *abort_flag != 0); };
        auto mma_done = [&]() -> bool {
            const bool ok = mbar_wait(&bar[B_MMA], ph & 1, abort_flag);
            ph++;
            fence_after_sync();
            const bool go = !wabort(ok);
            if (go) pending = false;
            return go;
        };
        const uint32_t sS = smem_u32(sm + OFF_S), sU = smem_u32(sm + OFF_U), sUD = smem_u32(sm + OFF_UD);
        float S[32];  // state row trow, value columns j0 + cb ... + 31
        {
            const float *s0 = a.S0 ? a.S0 + (((size_t)b * H + h) * DK + trow) * DV + j0 + cb : nullptr;
#pragma unroll
            for (int j = 0; j < 32; ++j) S[j] = s0 ? s0[j] : 0.f;
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) st_chunk(sm + OFF_S, swz(trow, hf * 4 + c4), S + c4 * 8);
        }
        fence_proxy_async();
        named_sync(2, 256);
        // o of the previous chunk is finished by lanes 64-127 while the next chunk starts: they
        // stage it in OFF_O and one of them issues its TMA store (rows past T are clipped).
        // Fused forward: y = o / sqrt(mean(o^2) + eps) w sigmoid(gate), the mean over all dv columns,
        // half of them in the partner CTA.  On the critical path (while the next chunk's first
        // product runs) only o is formed: the partial row sums of its squares and z = o sigmoid(gate) w
        // (bf16, in the buffer of the chunk's parity; lanes 0-63 turn the gate tile into
        // sigmoid(gate) meanwhile).  In the window where lanes 0-63 form U, lanes 64-127 keep the new chunk's
        // sigmoid(gate), add up the two column halves' sums of the chunk before and send them to
        // the partner's slot (chunk mod 4); while the second product runs, they finish y = z / rms
        // of the chunk two back, in place, and store it.  (The partner writes slot p mod 4 again for
        // chunk p + 4, which it reaches only after this CTA has sent its sums of chunk p + 3, i.e.
        // after y(p) is done here.)
        int prev_L = 0, prev_t0 = 0, prev_m = 0;
        float prev_eg = 0.f, inv_y = 0.f;
        uint32_t prev_buf = 0;
        uint32_t sg0[16] = {}, sg1[16] = {};  // fused, lanes 64-127: sigmoid(gate) of even / odd chunks (bf16 pairs)
        float loc_prev = 0.f;                 // fused: this CTA's full row sum of squares of the chunk before
        auto zbuf = [&](int par) -> unsigned char * { return sm + (par ? OFF_O1 : OFF_Y); };
        // fused: the partial row sums of squares of chunks of parity par, [2 column halves][64]
        auto sq_tile = [&](int par) -> float * {
            return reinterpret_cast<float *>(sm + OFF_MISC + (par ? M_SQ1 : M_SKP));
        };
        // fused: the inverse RMS of chunk q's row from this CTA's sums (loc_prev) and the partner's;
        // a wait that gives up raises the abort flag, which the next consensus acts on.  Once its
        // own wait is over, one thread arms the slot for chunk q + 4 (the partner sends those sums
        // only after this CTA has sent its sums of chunk q + 3, long after every wait on chunk q here).
        auto fused_inv = [&](int q) -> float {
            const float *xs = reinterpret_cast<const float *>(sm + OFF_MISC + M_XS);
            mbar_wait(&bar[B_XS0 + (q & 3)], (uint32_t)(q >> 2) & 1, abort_flag);
            if (ostore) mbar_arrive_tx(&bar[B_XS0 + (q & 3)], 64 * 4);
            return rsqrtf((loc_prev + xs[(q & 3) * 64 + trow - 64]) * (1.f / DV) + POST_EPS);
        };
        // fused: this CTA's row sums of chunk q (both column halves) into loc_prev, and to the partner
        auto send_sums = [&](int q) {
            const int r = trow - 64;
            const float *sq = sq_tile(q & 1);
            loc_prev = sq[r] + sq[64 + r];
            if (hf == 0) {
                const uint32_t partner = (uint32_t)half ^ 1u, slot = (uint32_t)q & 3;
                float *xs = reinterpret_cast<float *>(sm + OFF_MISC + M_XS);
                st_async_f32(map_to_rank(xs + slot * 64 + r, partner), loc_prev,
                             map_to_rank(&bar[B_XS0 + slot], partner));
            }
        };
        // fused: y of chunk q = z inv, in place in its buffer, then stored (lanes 64-127 together)
        auto y_step = [&](int q, float inv) {
            const int r = trow - 64;
            unsigned char *zb = zbuf(q & 1);
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                float z8[8];
                ld_chunk(zb, swz(r, hf * 4 + c4), z8);
#pragma unroll
                for (int e = 0; e < 8; ++e) z8[e] *= inv;
                st_chunk(zb, swz(r, hf * 4 + c4), z8);
            }
            fence_proxy_async();
            named_sync(3, 128);
            if (ostore) {
                tma_store_4d(&mp.y, zb, j0, h, q * C, b);
                bulk_commit();
            }
        };
        auto o_epilogue = [&]() {
            if (!OUT || trow < 64 || prev_L == 0 || (!FUSED && !a.has_out)) return;
            const int r = trow - 64;
            float d[32], p[32];
            tmem_row32(tl + TM_D + prev_buf, d);
            tmem_row32(tl + TM_D + prev_buf + 64, p);
#pragma unroll
            for (int j = 0; j < 32; ++j) d[j] = prev_eg * d[j] + p[j];
            if (FUSED) {
                float ss = 0.f;
#pragma unroll
                for (int j = 0; j < 32; ++j) ss += d[j] * d[j];
                sq_tile(prev_m & 1)[hf * 64 + r] = ss;
            }
            if (ostore) bulk_wait_read_all();  // the earlier stores have read their staging tiles
            named_sync(3, 128);
            if (a.has_out) {
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) st_chunk(sm + OFF_O, swz(r, hf * 4 + c4), d + c4 * 8);
            }
            if (FUSED) {  // z = o sigmoid(gate) w
                unsigned char *zb = zbuf(prev_m & 1);
                const float4 *wn4 = reinterpret_cast<const float4 *>(sm + OFF_MISC + M_WN) + cb / 4;
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const float4 w0 = wn4[c4 * 2], w1 = wn4[c4 * 2 + 1];
                    const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        const uint32_t sgw = (prev_m & 1) ? sg1[c4 * 4 + x] : sg0[c4 * 4 + x];
                        d[c4 * 8 + 2 * x] *= bf16_lo(sgw) * wv[2 * x];
                        d[c4 * 8 + 2 * x + 1] *= bf16_hi(sgw) * wv[2 * x + 1];
                    }
                    st_chunk(zb, swz(r, hf * 4 + c4), d + c4 * 8);
                }
            }
            fence_proxy_async();
            named_sync(3, 128);
            if (ostore && a.has_out) {
                tma_store_4d(&mp.out, sm + OFF_O, j0, h, prev_t0, b);
                bulk_commit();
            }
        };
        // fused: y of the last two chunks, after the loop (lanes 64-127 only)
        auto y_last = [&]() {
            if (prev_m >= 1) {
                if (ostore) bulk_wait_read_all();  // buffers of the earlier y stores
                named_sync(3, 128);
                y_step(prev_m - 1, fused_inv(prev_m - 1));
            }
            named_sync(3, 128);  // both column halves' sums of the last chunk are in place
            send_sums(prev_m);
            const float inv = fused_inv(prev_m);
            y_step(prev_m, inv);
        };
        for (int mi = 0; mi < NS; ++mi) {  // stages and phases by mi; m is the chunk of the sequence
            const int m = m0 + mi, s = mi & 1, t0 = m * C, L = min(C, T - t0);
            const uint32_t buf = (uint32_t)(mi & 1) * 128;
            const size_t ci = ci0 + m;
            unsigned char *st = sm + s * STAGE;
            const bool got = mbar_wait(&bar[B_FULL0 + s], (mi >> 1) & 1, abort_flag);
            if (wabort(got)) break;
            // this chunk's factors, read before the stage is released
            const float *cf = cf_all + s * 132;
            // KDA: this thread's state row decays by e^{g_C} of its key channel; no row factors
            const float egC = KDA ? cf[trow] : cf[128];
            const float rowf = KDA ? 1.f : cf[trow];  // lanes 0-63: e^{gC - g_r}; lanes 64-127: e^{g_r}, r = trow - 64
            // ---------------- D = [W ; q] S ----------------
            if (wc == 0) {
                fence_after_sync();
                bulk_wait_read_all();  // the previous chunk's U store has read OFF_U
                const uint32_t id = idesc_bf16(128, 64, 0, 1);
                const uint32_t swq = smem_u32(st + FS_WQ);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_bf16(tbase + TM_D + buf, sdesc(swq + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024),
                             sdesc(sS + k * 2048, 1024, 1024), id, k > 0);
                mma_commit(&bar[B_MMA]);
                if (KEEP) {  // the state entering chunk m, straight from its bf16 operand tile
                    tma_store_2d(&mp.Sn, sm + OFF_S, j0, (int)ci * DK);
                    bulk_commit();
                }
            }
            pending = true;
            o_epilogue();  // previous chunk, lanes 64-127
            if (FUSED && trow < 64) {
                // lanes 0-63, idle while D runs: this chunk's gate logits -> sigmoid(gate), in place
                // (bf16; row trow, this thread's 32 columns), read by lanes 64-127 after the next barrier
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    uint4 *gp = reinterpret_cast<uint4 *>(st + FS_G + swz(trow, hf * 4 + c4));
                    const uint4 g4 = *gp;
                    *gp = make_uint4(sigmoid_bf16x2(g4.x), sigmoid_bf16x2(g4.y), sigmoid_bf16x2(g4.z),
                                     sigmoid_bf16x2(g4.w));
                }
            }
            if (!mma_done()) break;
            // ---------------- U = U~ - W S;  U and e^{gC - g} U tiles ----------------
            if (trow < 64) {
                const int r = trow;
                float v[32];
                tmem_row32(tl + TM_D + buf, v);
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const uint32_t o = swz(r, hf * 4 + c4);
                    float ut[8];
                    ld_chunk(st + FS_UP, o, ut);
#pragma unroll
                    for (int e = 0; e < 8; ++e) ut[e] -= v[c4 * 8 + e];
                    st_chunk(sm + OFF_U, o, ut);
#pragma unroll
                    for (int e = 0; e < 8; ++e) ut[e] *= rowf;
                    st_chunk(sm + OFF_UD, o, ut);
                }
            } else if (FUSED) {
                // lanes 64-127, idle here: this chunk's sigmoid(gate), kept for its z; the inverse
                // RMS of the chunk two back; the previous chunk's row sums (its o epilogue just ran)
                // to the partner
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const uint4 g4 = *reinterpret_cast<const uint4 *>(st + FS_G + swz(trow - 64, hf * 4 + c4));
                    if (mi & 1) {
                        sg1[c4 * 4] = g4.x; sg1[c4 * 4 + 1] = g4.y; sg1[c4 * 4 + 2] = g4.z; sg1[c4 * 4 + 3] = g4.w;
                    } else {
                        sg0[c4 * 4] = g4.x; sg0[c4 * 4 + 1] = g4.y; sg0[c4 * 4 + 2] = g4.z; sg0[c4 * 4 + 3] = g4.w;
                    }
                }
                if (mi >= 2) inv_y = fused_inv(mi - 2);  // (the fused forward runs whole sequences: mi = m)
                if (mi >= 1) send_sums(mi - 1);
            }
            fence_proxy_async();
            fence_before_sync();
            if (wabort(true)) break;
            // ---------------- E = k^T (e^{gC-g} U);  O' = [* ; P] U;  U out ----------------
            if (wc == 0) {
                fence_after_sync();
                if (KEEP) tma_store_2d(&mp.Un, sm + OFF_U, j0, (int)ci * C);
                if (OUT && a.has_u) tma_store_4d(&mp.u, sm + OFF_U, j0, h, t0, b);
                if (KEEP || (OUT && a.has_u)) bulk_commit();
                const uint32_t sk = smem_u32(st + FS_K), sup = smem_u32(st + FS_UP);
                const uint32_t ide = idesc_bf16(128, 64, 1, 1), ido = idesc_bf16(128, 64, 0, 1);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16(tbase + TM_E, sdesc(sk + k * 2048, 8192, 1024), sdesc(sUD + k * 2048, 1024, 1024), ide,
                             k > 0);
                if (OUT) {
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mma_bf16(tbase + TM_D + buf + 64, sdesc(sup + k * 32, 16, 1024), sdesc(sU + k * 2048, 1024, 1024),
                                 ido, k > 0);
                }
                mma_commit(&bar[B_MMA]);
            }
            pending = true;
            if (KEEP && wc == 0) bulk_wait_read_1();  // the S_m store has read OFF_S
            if (FUSED && trow >= 64 && mi >= 2) y_step(mi - 2, inv_y);  // while the second product runs
            if (!mma_done()) break;
            if (wc == 0) mbar_arrive(&bar[B_EMPTY0 + s]);
            // ---------------- S <- e^{gC} S + E ----------------
            {
                float ev[32];
                tmem_row32(tl + TM_E, ev);
#pragma unroll
                for (int j = 0; j < 32; ++j) S[j] = egC * S[j] + ev[j];
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) st_chunk(sm + OFF_S, swz(trow, hf * 4 + c4), S + c4 * 8);
            }
            fence_proxy_async();
            fence_before_sync();
            if (wabort(true)) break;
            prev_L = L; prev_t0 = t0; prev_eg = rowf; prev_buf = buf; prev_m = mi;
        }
        // the last chunk (all chain threads agree first: the fused epilogue waits on the partner)
        const bool fin = !named_sync_any(2, 256, *abort_flag != 0);
        if (fin) o_epilogue();
        if (FUSED && fin && trow >= 64 && prev_L > 0 && !named_sync_any(3, 128, *abort_flag != 0)) y_last();
        if (wc == 0 || ostore) bulk_wait_all();
        if (*abort_flag == 0) {
            if (OUT && a.ST) {
                float *dst = a.ST + (((size_t)b * H + h) * DK + trow) * DV + j0 + cb;
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    *reinterpret_cast<float4 *>(dst + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
            }
        } else if (pending) {
            volatile int dummy = 0;
            mbar_wait(&bar[B_MMA], ph & 1, &dummy, 100000000ull);
        }
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (FUSED) cluster_sync();  // no CTA leaves while its partner may still reach its shared memory
    if (warp == 0) tmem_dealloc(tbase, 512);
}

// ====================================== reverse chain ======================================
// KDA: q and k arrive gate-scaled (q e^g, k e^{g_C - g}, as in the forward), so the row
// factors are 1 and dS decays by row.
template <int KDA>
__global__ void __launch_bounds__(NTHREADS, 1) k_chain_rev(const __grid_constant__ RMaps mp, Args a) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + OFF_MISC + M_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC + M_TMEM);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + OFF_MISC + M_ABORT);
    float *cf_all = reinterpret_cast<float *>(sm + OFF_MISC + M_CF);
    float *skp = reinterpret_cast<float *>(sm + OFF_MISC + M_SKP);

    const int half = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int j0 = half * DVB;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = a.H, N = a.N;
    const int M1 = a.m1 > 0 ? a.m1 : N, NS = M1 - a.m0;  // this launch's chunks [m0, M1), last first
    const size_t ci0 = ((size_t)b * H + h) * N;

    if (threadIdx.x == 0) {
        for (int i = 0; i < B_NUM; ++i) mbar_init(&bar[i], (i == B_FULL0 || i == B_FULL1) ? 2 : 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, 256);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = *tmem_slot;

    if (warp == 0) {
        // ================================ producer ================================
        int issued[2] = {0, 0};
        FactorIn fin;
        for (int m = 0; m < NS; ++m) {
            const int mc = M1 - 1 - m, s = m & 1, t0 = mc * C;
            const int ci = (int)(ci0 + mc);
            factors_fetch<KDA != 0, false>(a, (size_t)ci, lane, fin);
            if (m >= 2 && !mbar_wait(&bar[B_EMPTY0 + s], ((m >> 1) - 1) & 1, abort_flag)) break;
            unsigned char *st = sm + s * STAGE;
            if (lane == 0) {
                mbar_arrive_tx(&bar[B_FULL0 + s], 73728u + (a.has_du ? 8192u : 0u));
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    if (KDA) {
                        tma_load_2d(st + RS_K + p * 8192, &mp.k, 64 * p, ci * C, &bar[B_FULL0 + s]);
                        tma_load_2d(st + RS_Q + p * 8192, &mp.q, 64 * p, ci * C, &bar[B_FULL0 + s]);
                    } else {
                        tma_load_4d(st + RS_K + p * 8192, &mp.k, 64 * p, h, t0, b, &bar[B_FULL0 + s]);
                        tma_load_4d(st + RS_Q + p * 8192, &mp.q, 64 * p, h, t0, b, &bar[B_FULL0 + s]);
                    }
                    tma_load_2d(st + RS_W + p * 8192, &mp.W, 64 * p, ci * C, &bar[B_FULL0 + s]);
                }
                tma_load_4d(st + RS_DO, &mp.dout, j0, h, t0, b, &bar[B_FULL0 + s]);
                tma_load_2d(st + RS_P, &mp.P, 0, ci * C, &bar[B_FULL0 + s]);
                if (a.has_du) tma_load_4d(st + RS_DX, &mp.du, j0, h, t0, b, &bar[B_FULL0 + s]);
                tma_load_2d(st + RS_UN, &mp.Un, j0, ci * C, &bar[B_FULL0 + s]);
            }
            factors_store<KDA != 0, false>(fin, cf_all + s * 132, lane);
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[B_FULL0 + s]);
            issued[s]++;
        }
        if (*abort_flag) {
            volatile int dummy = 0;
            for (int s = 0; s < 2; ++s)
                if (issued[s] > 0) mbar_wait(&bar[B_FULL0 + s], (issued[s] - 1) & 1, &dummy, 100000000ull);
        }
    } else {
        // ================================ chain ================================
        const ChainLane cl(warp, lane);
        const int wc = cl.wc, trow = cl.trow, hf = cl.hf, cb = cl.cb;
        const uint32_t tl = tbase + ((uint32_t)(cl.q4 * 32) << 16) + (uint32_t)cb;
        constexpr uint32_t TM_A = 0, TM_B = 64, TM_P = 128;
        uint32_t ph = 0;
        bool pending = false;
        auto wabort = [&](bool ok) -> bool { return named_sync_any(2, 256, !ok || *abort_flag != 0); };
        auto mma_done = [&]() -> bool {
            const bool ok = mbar_wait(&bar[B_MMA], ph & 1, abort_flag);
            ph++;
            fence_after_sync();
            const bool go = !wabort(ok);
            if (go) pending = false;
            return go;
        };
        const uint32_t sS = smem_u32(sm + OFF_S), sU = smem_u32(sm + OFF_U);
        float S[32];  // dL/dS of the state leaving the current chunk: row trow, columns j0 + cb ...
        {
            const float *s0 = a.S0 ? a.S0 + (((size_t)b * H + h) * DK + trow) * DV + j0 + cb : nullptr;
#pragma unroll
            for (int j = 0; j < 32; ++j) S[j] = s0 ? s0[j] : 0.f;
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) st_chunk(sm + OFF_S, swz(trow, hf * 4 + c4), S + c4 * 8);
        }
        fence_proxy_async();
        named_sync(2, 256);
        for (int m = 0; m < NS; ++m) {
            const int mc = M1 - 1 - m, s = m & 1;
            const size_t ci = ci0 + mc;
            unsigned char *st = sm + s * STAGE;
            const bool got = mbar_wait(&bar[B_FULL0 + s], (m >> 1) & 1, abort_flag);
            if (wabort(got)) break;
            const float *cf = cf_all + s * 132;
            const float egC = KDA ? cf[trow] : cf[128];  // KDA: this thread's state row decays by its channel
            // ------- D_a = k dS+, D_p = P^T dO  (M = 128: rows 64..127 discarded) -------
            if (wc == 0) {
                fence_after_sync();
                bulk_wait_read_all();  // the previous chunk's dU store has read OFF_U
                const uint32_t id = idesc_bf16(128, 64, 0, 1), idp = idesc_bf16(128, 64, 1, 1);
                const uint32_t sk = smem_u32(st + RS_K), sp = smem_u32(st + RS_P), sdo = smem_u32(st + RS_DO);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_bf16(tbase + TM_A, sdesc(sk + (k >> 2) * 8192 + (k & 3) * 32, 16, 1024),
                             sdesc(sS + k * 2048, 1024, 1024), id, k > 0);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16(tbase + TM_P, sdesc(sp + k * 2048, 8192, 1024), sdesc(sdo + k * 2048, 1024, 1024), idp,
                             k > 0);
                mma_commit(&bar[B_MMA]);
                tma_store_2d(&mp.dSn, sm + OFF_S, j0, (int)ci * DK);  // dS_{n+1} from its operand tile
                bulk_commit();
            }
            pending = true;
            if (!mma_done()) break;
            // ---------------- dU = du + P^T dO + diag(e^{gC - g}) D_a;  U_r . (Kbar dS+)_r ----------------
            if (trow < 64) {
                const int r = trow;
                const float f = KDA ? 1.f : cf[r];
                float v[32], pd[32], rs = 0.f;
                tmem_row32(tl + TM_A, v);
                tmem_row32(tl + TM_P, pd);
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const uint32_t o = swz(r, hf * 4 + c4);
                    float d[8], x[8], un[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) d[e] = pd[c4 * 8 + e];
                    ld_chunk(st + RS_UN, o, un);
                    if (a.has_du) {
                        ld_chunk(st + RS_DX, o, x);
#pragma unroll
                        for (int e = 0; e < 8; ++e) d[e] += x[e];
                    }
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float kd = f * v[c4 * 8 + e];
                        rs += un[e] * kd;
                        d[e] += kd;
                    }
                    st_chunk(sm + OFF_U, o, d);
                }
                skp[hf * 64 + r] = rs;
            } else if (!KDA) {
                // lanes 64-127: q rows scaled by e^{g_r} (for q^T diag(e^g) dO)
                for (int x = (cl.q4 - 2) * 32 + lane + hf * 64; x < 1024; x += 128) {  // 128 threads
                    float v[8];
                    ld_chunk(st + RS_Q, (uint32_t)x * 16, v);
                    const float f = cf[64 + ((x >> 3) & 63)];
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[e] *= f;
                    st_chunk(st + RS_Q, (uint32_t)x * 16, v);
                }
            }
            fence_proxy_async();
            fence_before_sync();
            if (wabort(true)) break;
            if (trow < 64 && hf == 0) a.skt[ci * 2 * C + half * C + trow] = skp[trow] + skp[64 + trow];
            // ---------------- D_b = (diag(e^g) q)^T dO - W^T dU;  dU out ----------------
            if (wc == 0) {
                fence_after_sync();
                const uint32_t idb = idesc_bf16(128, 64, 1, 1), id = idesc_bf16(128, 64, 1, 1, 1);
                const uint32_t sq = smem_u32(st + RS_Q), sdo = smem_u32(st + RS_DO), sw = smem_u32(st + RS_W);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16(tbase + TM_B, sdesc(sq + k * 2048, 8192, 1024), sdesc(sdo + k * 2048, 1024, 1024), idb,
                             k > 0);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_bf16(tbase + TM_B, sdesc(sw + k * 2048, 8192, 1024), sdesc(sU + k * 2048, 1024, 1024), id, 1);
                mma_commit(&bar[B_MMA]);
                tma_store_2d(&mp.dUn, sm + OFF_U, j0, (int)ci * C);
                bulk_commit();
                bulk_wait_read_1();  // the dS_{n+1} store has read OFF_S
            }
            pending = true;
            if (!mma_done()) break;
            if (wc == 0) mbar_arrive(&bar[B_EMPTY0 + s]);
            // ---------------- dS_n = e^{gC} dS+ + D_b ----------------
            {
                float dv[32];
                tmem_row32(tl + TM_B, dv);
#pragma unroll
                for (int j = 0; j < 32; ++j) S[j] = egC * S[j] + dv[j];
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) st_chunk(sm + OFF_S, swz(trow, hf * 4 + c4), S + c4 * 8);
            }
            fence_proxy_async();
            fence_before_sync();
            if (wabort(true)) break;
        }
        if (wc == 0) bulk_wait_all();
        if (*abort_flag == 0) {
            if (a.ST) {
                float *dst = a.ST + (((size_t)b * H + h) * DK + trow) * DV + j0 + cb;
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    *reinterpret_cast<float4 *>(dst + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
            }
        } else if (pending) {
            volatile int dummy = 0;
            mbar_wait(&bar[B_MMA], ph & 1, &dummy, 100000000ull);
        }
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == 0) tmem_dealloc(tbase, 256);
}

}  // namespace tch

bool tc_split_supported(const Geo &g, bool bf16) {
    return bf16 && g.C == 64 && g.dk == 128 && g.dv == 128 && g.variant != VAR_KDA &&
           (size_t)g.B * g.H * g.N * 128 <= (size_t)INT_MAX;
}

bool tc_split_kda_supported(const Geo &g, bool bf16) {
    return bf16 && g.C == 64 && g.dk == 128 && g.dv == 128 && g.variant == VAR_KDA &&
           (size_t)g.B * g.H * g.N * KDA_KH_ROWS <= (size_t)INT_MAX;
}

static size_t ws_al256(size_t x) { return (x + 255) & ~(size_t)255; }

// Carves the given parts of the split-path workspace from base (or only counts, when base
// is null); returns the bytes they span.
static size_t ws_carve(const Geo &g, int parts, char *base, TcWs *w) {
    const size_t nc = (size_t)g.B * g.H * g.N, C = g.C, DK = g.dk, DV = g.dv;
    size_t off = 0;
    auto take = [&](size_t bytes) { char *r = base ? base + off : nullptr; off += ws_al256(bytes); return r; };
    if (parts & WS_FWD) {
        w->gb = (float *)take(nc * 2 * C * 4);
        w->W = (__nv_bfloat16 *)take(nc * C * DK * 2);
        w->Ut = (__nv_bfloat16 *)take(nc * C * DV * 2);
        w->P = (__nv_bfloat16 *)take(nc * C * C * 2);
    }
    if (parts & WS_KEEP) {
        w->Tn = (__nv_bfloat16 *)take(nc * C * C * 2);
        w->KK = (__nv_bfloat16 *)take(nc * C * C * 2);
    }
    if (parts & WS_STATE) {
        w->Sn = (__nv_bfloat16 *)take(nc * DK * DV * 2);
        w->Un = (__nv_bfloat16 *)take(nc * C * DV * 2);
    }
    if (parts & WS_REV) {
        w->dSn = (__nv_bfloat16 *)take(nc * DK * DV * 2);
        w->dUn = (__nv_bfloat16 *)take(nc * C * DV * 2);
        w->skt = (float *)take(nc * 2 * C * 4);
    }
    if (parts & WS_KDA) {
        __nv_bfloat16 **tiles[] = {&w->Kt1, &w->Qt1, &w->Kt};
        for (__nv_bfloat16 **t : tiles) *t = (__nv_bfloat16 *)take(nc * C * DK * 2);
        w->Kh = (__nv_bfloat16 *)take(nc * KDA_KH_ROWS * DK * 2);
        w->Dx = (float *)take(nc * 2 * C * 16 * 4);
    }
    if (parts & WS_KDAC) {
        w->Qt = (__nv_bfloat16 *)take(nc * C * DK * 2);
        w->Kb = (__nv_bfloat16 *)take(nc * C * DK * 2);
        w->egc = (float *)take(nc * DK * 4);
        w->kwide = (int *)take(nc * 4);
    }
    if (parts & WS_KDAG) w->G = (float *)take(nc * C * DK * 4);
    if (parts & WS_RN) w->rn = (float *)take(nc * 2 * C * 4);
    return off;
}

size_t tc_ws_bytes(const Geo &g, int parts) {
    TcWs w = {};
    return ws_carve(g, parts, nullptr, &w);
}

void tc_ws_carve(const Geo &g, int parts, void *base, TcWs *w) { ws_carve(g, parts, (char *)base, w); }

cudaError_t tc_chain_fwd(const Geo &g, const Tensors &t, const TcWs &w, int mode, cudaStream_t s, Rec &rec) {
    using namespace tch;
    FMaps mp;
    const uint64_t Bn = g.B, T = g.T, H = g.H, NC = (uint64_t)g.B * g.H * g.N;
    const bool out = mode != 1, keep = mode == 1 || mode == 2, kda = g.variant == VAR_KDA, fused = mode == 3;
    if (fused && (kda || !t.y || !t.gate_o || !t.w_norm || !w.rn)) return cudaErrorInvalidValue;
    bool ok = (kda ? tc::make_map_2d_bf16(&mp.q, w.Qt, DK, NC * C, 64) && tc::make_map_2d_bf16(&mp.k, w.Kb, DK, NC * C, 64)
                   : tc::make_map_4d_bf16(&mp.q, t.q, DK, H, T, Bn, 64) &&
                         tc::make_map_4d_bf16(&mp.k, t.k, DK, H, T, Bn, 64)) &&
              tc::make_map_2d_bf16(&mp.W, w.W, DK, NC * C, 64) && tc::make_map_2d_bf16(&mp.Ut, w.Ut, DV, NC * C, 64) &&
              tc::make_map_2d_bf16(&mp.P, w.P, C, NC * C, 64);
    mp.out = mp.u = mp.Sn = mp.Un = mp.gate = mp.y = mp.q;  // unused ones keep a valid map
    if (ok && fused)
        ok = tc::make_map_4d_bf16(&mp.gate, t.gate_o, DV, H, T, Bn, 64) && tc::make_map_4d_bf16(&mp.y, t.y, DV, H, T, Bn, 64);
    if (ok && keep)
        ok = tc::make_map_2d_bf16(&mp.Sn, w.Sn, DV, NC * DK, 128) && tc::make_map_2d_bf16(&mp.Un, w.Un, DV, NC * C, 64);
    if (ok && out && t.out) ok = tc::make_map_4d_bf16(&mp.out, t.out, DV, H, T, Bn, 64);
    if (ok && out && t.u) ok = tc::make_map_4d_bf16(&mp.u, t.u, DV, H, T, Bn, 64);
    if (!ok) return cudaErrorInvalidValue;
    Args a = {};
    a.gb = w.gb; a.B = g.B; a.T = g.T; a.H = g.H; a.N = g.N;
    a.S0 = t.S0; a.egc = w.egc; a.rn = w.rn; a.wn = t.w_norm; a.m0 = w.m0; a.m1 = w.m1;
    if (out) {
        a.has_out = t.out != nullptr; a.has_u = t.u != nullptr; a.ST = t.S_T;
    }
    const size_t smem = SMEM_BYTES + 1024;
    const dim3 grid(DV / DVB, g.H, g.B);
    cudaError_t e;
    auto go = [&](auto kern) -> cudaError_t {
        cudaError_t e2 = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e2 != cudaSuccess) return e2;
        rec.mark(s);
        if (!fused) {
            kern<<<grid, NTHREADS, smem, s>>>(mp, a);
            return cudaSuccess;
        }
        // the two value halves of a (b, h) form a cluster (they exchange the output's row sums)
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = grid;
        cfg.blockDim = dim3(NTHREADS);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, kern, mp, a);
    };
    if (kda) e = mode == 0 ? go(k_chain_fwd<0, 1>) : mode == 1 ? go(k_chain_fwd<1, 1>) : go(k_chain_fwd<2, 1>);
    else if (mode == 0) e = go(k_chain_fwd<0, 0>);
    else if (mode == 1) e = go(k_chain_fwd<1, 0>);
    else if (mode == 2) e = go(k_chain_fwd<2, 0>);
    else e = go(k_chain_fwd<3, 0>);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t tc_chain_rev(const Geo &g, const Tensors &t, const TcWs &w, cudaStream_t s, Rec &rec) {
    using namespace tch;
    RMaps mp;
    const uint64_t Bn = g.B, T = g.T, H = g.H, NC = (uint64_t)g.B * g.H * g.N;
    const bool kda = g.variant == VAR_KDA;
    const bool ok = (kda ? tc::make_map_2d_bf16(&mp.q, w.Qt, DK, NC * C, 64) && tc::make_map_2d_bf16(&mp.k, w.Kb, DK, NC * C, 64)
                         : tc::make_map_4d_bf16(&mp.q, t.q, DK, H, T, Bn, 64) &&
                               tc::make_map_4d_bf16(&mp.k, t.k, DK, H, T, Bn, 64)) &&
                    tc::make_map_4d_bf16(&mp.dout, t.dout, DV, H, T, Bn, 64) &&
                    tc::make_map_2d_bf16(&mp.W, w.W, DK, NC * C, 64) && tc::make_map_2d_bf16(&mp.P, w.P, C, NC * C, 64) &&
                    tc::make_map_2d_bf16(&mp.Un, w.Un, DV, NC * C, 64) && tc::make_map_2d_bf16(&mp.dUn, w.dUn, DV, NC * C, 64) &&
                    tc::make_map_2d_bf16(&mp.dSn, w.dSn, DV, NC * DK, 128) &&
                    (t.du ? tc::make_map_4d_bf16(&mp.du, t.du, DV, H, T, Bn, 64) : (mp.du = mp.dout, true));
    if (!ok) return cudaErrorInvalidValue;
    Args a = {};
    a.gb = w.gb; a.B = g.B; a.T = g.T; a.H = g.H; a.N = g.N;
    a.S0 = t.dS_T; a.ST = t.dS0; a.skt = w.skt; a.has_du = t.du != nullptr; a.egc = w.egc;
    a.m0 = w.m0; a.m1 = w.m1;
    const size_t smem = SMEM_BYTES + 1024;
    auto go = [&](auto kern) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        rec.mark(s);
        kern<<<dim3(DV / DVB, g.H, g.B), NTHREADS, smem, s>>>(mp, a);
        return cudaGetLastError();
    };
    return kda ? go(k_chain_rev<1>) : go(k_chain_rev<0>);
}

}  // namespace dr
