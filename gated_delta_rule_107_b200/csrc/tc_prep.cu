// tc_prep.cu -- the per-chunk products of the chunked gated delta rule, one CTA per chunk
// (Gated DeltaNet, DeltaNet and KDA; bf16 I/O, dk = dv = 128, C = 64).
//
// Chunked form of "线性注意力架构演进与Kimi Delta Attention创新实践" (sections 2.1, 6.1,
// 6.2, 7.1).  With g the in-chunk cumulative log gate:
//
//   P1   [k ; q] . k^T                        -> k.k^T (rows 0-63), q.k^T (rows 64-127)
//        A = beta_r e^{g_r - g_i} k_r.k_i (i < r),   P = e^{g_r - g_i} q_r.k_i (i <= r)
//   T  = (I + A)^-1                            (the UT transform; tc_inverse.cuh)
//   W  = T diag(beta e^g) k,   U~ = T diag(beta) v
//   backward (and a forward that saves for it): T and k k^T kept for the gradient kernel.
// KDA's gates are per key channel, so they cannot leave the dot products as scalars: a
// first kernel (k_kda_gates) writes the gate-scaled operands.  The pair factor of row r and
// column i <= r is split at the first token b = 16 floor(r / 16) of r's 16-token block,
// e^{g_r - g_i} = e^{g_r - g_b} e^{g_b - g_i} (log-space gates, section 7.1; second-level
// blocking, section 2.2): the row factor is <= 1, and so is the column factor for every i
// before the block.  Each block of rows has its own column operand, so P1 becomes one N = 160
// product against the four column operands stacked,
//   P1 = [k e^{g - g_b} ; q e^{g - g_b}] . [K_0 ; K_1 ; K_2 ; K_3]^T,   K_R = k_i e^{g_16R - g_i}
// (i = 0 .. 16 R + 15), of which row r reads the section of its block; W = T diag(beta) (k e^g).
// Inside a block the column factor is at most e^{the block's fall}; a chunk where some channel
// falls by more than KDA_DIAG_SPAN inside a block takes its in-block entries from exact
// per-pair sums instead (k_kda_diag).
//
// Every chunk is independent, so the grid covers all chunks of all heads at once (two
// CTAs per SM); the serial state chains (tc_chain.cu) then only carry the state.  The
// products leave as bf16 tiles through TMA stores (W, U~, P, and T, k k^T from tiles freed by
// then), and g, beta as fp32.  The products with 64 rows use M = 128 MMAs whose rows 64..127 read
// other (valid) shared memory and are discarded.
#include "tc_host.cuh"
#include "tc_inverse.cuh"
#include "tc_path.cuh"
#include "tc_ptx.cuh"
#include "tc_tile.cuh"

namespace dr {
namespace tcp {

using namespace dr::tc;
using dr::tcf::ld_chunk;
using dr::tcf::st_chunk;
using dr::tcf::tmem_row64;

constexpr int C = 64, DK = 128, DV = 128;
constexpr int NTHREADS = 128;
// shared memory (bytes from a 1024-aligned base)
constexpr uint32_t OFF_KQ = 0;         // 32K [k_p0 | q_p0 | k_p1 | q_p1]; after P1: q_p0 -> k k^T (KEEP),
                                       //     then T diag(beta); q_p1 -> inverse scratch, then T diag(beta e^g)
constexpr uint32_t OFF_V = 32768;      // 16K v [i][j]
constexpr uint32_t OFF_F = 49152;      // 32K fp32 A | T (inverse), then staging W [r][c] | U~ [r][j]
constexpr uint32_t OFF_P = 81920;      //  8K P [r][i]
constexpr uint32_t OFF_MISC = 90112;   //  2K
constexpr uint32_t OFF_X = 92160;      // 16K KDA: k e^g (W's B)
constexpr uint32_t OFF_KH = OFF_F;     // 40K KDA: P1's stacked B (two panels of 160 rows), over F and P
constexpr uint32_t KH_PANEL = KDA_KH_ROWS * 128;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 2048, SMEM_KDA = OFF_X + 16384;
static_assert(OFF_P == OFF_F + 32768 && OFF_KH + 2 * KH_PANEL <= OFF_MISC, "the KDA B operand spans F and P");
// misc
constexpr uint32_t M_BAR = 0;          // [0] loads, [1] MMA
constexpr uint32_t M_TMEM = 64, M_ABORT = 68, M_BIG = 72;
constexpr uint32_t M_PF = 256;         // gate factors [6][64]
enum { PF_GC = 0, PF_ROWP, PF_COLA, PF_BV, PF_BK, PF_RNK, PF_RNQ, PF_NUM };
static_assert(M_PF + PF_NUM * 256 <= 2048, "misc overflow");
// TMEM columns
constexpr uint32_t TM_G1 = 0, TM_XW = 0, TM_XU = 128, TM_COLS = 256;

struct Maps {
    CUtensorMap q, k, v;  // [B, T, H, 128] bf16; box 64 channels x 64 tokens
    CUtensorMap W, Ut;    // [chunks * 64][128] bf16; box 64 x 64 (stores)
    CUtensorMap P;        // [chunks * 64][64] bf16; box 64 x 64 (store)
    CUtensorMap KK, Tn;   // [chunks * 64][64] bf16; box 64 x 64 (stores, when KEEP)
    CUtensorMap Kt1, Qt1, Kt;  // KDA: [chunks * 64][128] bf16 gate-scaled operands; box 64 x 64
    CUtensorMap Kh;            // KDA: [chunks * 160][128] bf16; box 64 x 160
};

struct Args {
    const void *alpha, *beta;       // bf16 [B, T, H] (RAW: the raw forget and write-strength logits)
    float *gb;                      // [chunks][2][64]: g, beta
    float *rn;                      // RAW: [chunks][2][64] 1 / |k_r|, 1 / |q_r|
    const int *kwide;               // KDA: [chunks] in-block sums from Dx
    const float *Dx;                // KDA: [chunks][2][64][16]
    int B, T, H, N;
    int wave;                       // CTAs resident at once (2 per SM): the L2 prefetch distance
    int n0;                         // chunk of blockIdx.x = 0 (a launch may cover chunks n0 ..)
};

// L2 prefetch of a tiled box (no shared memory, nothing to wait for; a box outside the tensor
// fetches nothing)
__device__ __forceinline__ void l2_prefetch_2d(const CUtensorMap *map, int c0, int c1) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1)
                 : "memory");
}
__device__ __forceinline__ void l2_prefetch_4d(const CUtensorMap *map, int c0, int c1, int c2, int c3) {
    asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1), "r"(c2), "r"(c3)
                 : "memory");
}

// first column of block R's section of the KDA product (16 R (R + 1) / 2)
__host__ __device__ constexpr uint32_t kda_sec(int R) { return (uint32_t)(8 * R * (R + 1)); }

__device__ __forceinline__ float sigmoid_f(float x) { return 1.f / (1.f + __expf(-x)); }
// softplus(x) = max(x, 0) + log(1 + e^{-|x|}), finite for every x
__device__ __forceinline__ float softplus_f(float x) { return fmaxf(x, 0.f) + log1pf(__expf(-fabsf(x))); }
constexpr float PRE_EPS = 1e-6f;  // q_hat = q / sqrt(|q|^2 + eps), as the standalone pre-operation

// KEEP: also store T and k k^T (for the backward).  RAW: the fused pre-operation (KDA page
// section 7.1): q, k arrive as raw projections and are normalised through per-row factors
// (1/|k_i| joins the column factors of A and P and the row factor of W's operand), the gate
// and beta as raw logits (log alpha = -softplus(a), beta = sigmoid(b)).
template <int VAR, int KEEP, int RAW>
__global__ void __launch_bounds__(NTHREADS, 2) k_chunk_prep(const __grid_constant__ Maps mp, Args a) {
    static_assert(!RAW || (VAR != VAR_KDA && !KEEP), "the fused pre-operation serves the scalar-gate forward");
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    unsigned char *misc = sm + OFF_MISC;
    uint64_t *bar = reinterpret_cast<uint64_t *>(misc + M_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + M_TMEM);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + M_ABORT);
    volatile int *bigflag = reinterpret_cast<volatile int *>(misc + M_BIG);
    float *pf = reinterpret_cast<float *>(misc + M_PF);

    const int n = a.n0 + (int)blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int T = a.T, H = a.H, t0 = n * C, L = min(C, T - t0);
    const int ci = (b * H + h) * a.N + n;  // ci * 160 < 2^31 (checked by the launcher)
    const int trow = tid;                  // TMEM lane of this thread

    int mma_issued = 0;
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        *abort_flag = 0;
        fence_mbar_init();
        mbar_arrive_tx(&bar[0], VAR == VAR_KDA ? 65536u + 2 * KH_PANEL : 49152u);
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            if (VAR == VAR_KDA) {  // the gate-scaled operands of tc_kda_gates
                tma_load_2d(sm + OFF_KQ + p * 16384, &mp.Kt1, 64 * p, ci * C, &bar[0]);
                tma_load_2d(sm + OFF_KQ + p * 16384 + 8192, &mp.Qt1, 64 * p, ci * C, &bar[0]);
                tma_load_2d(sm + OFF_KH + p * KH_PANEL, &mp.Kh, 64 * p, ci * KDA_KH_ROWS, &bar[0]);
                tma_load_2d(sm + OFF_X + p * 8192, &mp.Kt, 64 * p, ci * C, &bar[0]);
            } else {
                tma_load_4d(sm + OFF_KQ + p * 16384, &mp.k, 64 * p, h, t0, b, &bar[0]);
                tma_load_4d(sm + OFF_KQ + p * 16384 + 8192, &mp.q, 64 * p, h, t0, b, &bar[0]);
            }
            tma_load_4d(sm + OFF_V + p * 8192, &mp.v, 64 * p, h, t0, b, &bar[0]);
        }
        // the inputs of the CTA that starts one wave later (CTAs are dispatched in launch order),
        // into L2 while this one computes: its loads then wait on L2 rather than HBM
        const long long lin = blockIdx.x + (long long)gridDim.x * (blockIdx.y + (long long)gridDim.y * blockIdx.z);
        const long long nx = lin + a.wave;
        if (a.wave > 0 && nx < (long long)gridDim.x * gridDim.y * gridDim.z) {
            const int n2 = a.n0 + (int)(nx % gridDim.x), h2 = (int)((nx / gridDim.x) % gridDim.y),
                      b2 = (int)(nx / ((long long)gridDim.x * gridDim.y));
            const int ci2 = (b2 * H + h2) * a.N + n2;
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                if (VAR == VAR_KDA) {
                    l2_prefetch_2d(&mp.Kt1, 64 * p, ci2 * C);
                    l2_prefetch_2d(&mp.Qt1, 64 * p, ci2 * C);
                    l2_prefetch_2d(&mp.Kh, 64 * p, ci2 * KDA_KH_ROWS);
                    l2_prefetch_2d(&mp.Kt, 64 * p, ci2 * C);
                } else {
                    l2_prefetch_4d(&mp.k, 64 * p, h2, n2 * C, b2);
                    l2_prefetch_4d(&mp.q, 64 * p, h2, n2 * C, b2);
                }
                l2_prefetch_4d(&mp.v, 64 * p, h2, n2 * C, b2);
            }
        }
    }
    if (warp == 0) tmem_alloc(tmem_slot, TM_COLS);
    if (warp == 1) {
        // in-chunk cumulative log gate (lane owns rows lane and lane + 32) and the factors
        float lg[2], bt[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int r = lane + 32 * hh;
            const size_t row = ((size_t)b * T + t0 + r) * H + h;
            lg[hh] = 0.f;
            bt[hh] = 0.f;
            if (r < L) {
                if (VAR == VAR_GATED) lg[hh] = RAW ? -softplus_f(tcf::bf(a.alpha, row)) : tcf::bf(a.alpha, row);
                bt[hh] = RAW ? sigmoid_f(tcf::bf(a.beta, row)) : tcf::bf(a.beta, row);
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
        const float gm = __shfl_sync(0xffffffffu, x0, 31);  // midpoint of the chunk
        float dev = fmaxf(fabsf(x0 - gm), fabsf(x1 - gm));
        dev = fmaxf(dev, __shfl_xor_sync(0xffffffffu, dev, 16));
        dev = fmaxf(dev, __shfl_xor_sync(0xffffffffu, dev, 8));
        dev = fmaxf(dev, __shfl_xor_sync(0xffffffffu, dev, 4));
        dev = fmaxf(dev, __shfl_xor_sync(0xffffffffu, dev, 2));
        dev = fmaxf(dev, __shfl_xor_sync(0xffffffffu, dev, 1));
        const float xs[2] = {x0, x1};
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int r = lane + 32 * hh;
            const float x = xs[hh];
            pf[PF_GC * 64 + r] = x;
            pf[PF_ROWP * 64 + r] = __expf(x - gm);
            pf[PF_COLA * 64 + r] = __expf(gm - x);
            pf[PF_BV * 64 + r] = bt[hh];
            pf[PF_BK * 64 + r] = bt[hh] * __expf(x);
            a.gb[(size_t)ci * 2 * C + r] = x;
            a.gb[(size_t)ci * 2 * C + C + r] = bt[hh];
        }
        if (lane == 0) *bigflag = dev > 80.f;
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tl = tbase + ((uint32_t)(warp * 32) << 16);
    auto sync = [&]() { named_sync(1, NTHREADS); };
    auto consensus = [&](bool ok) -> bool { return !named_sync_any(1, NTHREADS, !ok || *abort_flag != 0); };
    uint32_t ph = 0;
    auto wait_mma = [&]() -> bool {
        const bool ok = mbar_wait(&bar[1], ph & 1, abort_flag);
        ph++;
        fence_after_sync();
        return ok;
    };
    float *Asc = reinterpret_cast<float *>(sm + OFF_F);
    float *Tf = Asc + 4096;
    const uint32_t skq = smem_u32(sm + OFF_KQ), sv = smem_u32(sm + OFF_V);

    bool ok = consensus(mbar_wait(&bar[0], 0, abort_flag));
    // ---------------- P1: [k ; q] . k^T (KDA: against the four stacked sections) ----------------
    if (ok && tid == 0) {
        const uint32_t id = idesc_bf16(128, VAR == VAR_KDA ? KDA_KH_ROWS : 64, 0, 0);
        const uint32_t skh = smem_u32(sm + OFF_KH);
#pragma unroll
        for (int st = 0; st < 8; ++st) {
            const uint32_t ad = skq + (st >> 2) * 16384 + (st & 3) * 32;
            const uint32_t bd = VAR == VAR_KDA ? skh + (st >> 2) * KH_PANEL + (st & 3) * 32 : ad;
            mma_bf16(tbase + TM_G1, sdesc(ad, 16, 1024), sdesc(bd, 16, 1024), id, st > 0);
        }
        mma_commit(&bar[1]);
        mma_issued++;
    }
    if (RAW && ok) {  // while P1 runs: 1 / sqrt(|x|^2 + eps) of k row tid (tid < 64) or q row tid - 64
        const int r = trow & 63;
        const uint32_t base = OFF_KQ + (trow < 64 ? 0u : 8192u);
        float ss = 0.f;
#pragma unroll
        for (int p = 0; p < 2; ++p)
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                float x[8];
                ld_chunk(sm + base + p * 16384, swz(r, ch), x);
#pragma unroll
                for (int e = 0; e < 8; ++e) ss += x[e] * x[e];
            }
        const float rn = rsqrtf(ss + PRE_EPS);
        pf[(trow < 64 ? PF_RNK : PF_RNQ) * 64 + r] = rn;
        a.rn[(size_t)ci * 2 * C + (trow < 64 ? 0 : C) + r] = rn;
    }
    if (ok) ok = consensus(wait_mma());
    // ---------------- A (fp32, for the inverse), P (bf16 tile), k k^T ----------------
    if (ok) {
        float g1[64];
        if (VAR == VAR_KDA) {
            // lanes 0-15 of this warp hold rows of block R0, lanes 16-31 of block R0 + 1; each
            // reads columns i = 0 .. 16 R + 15 of its block's section (the rest of the row is 0)
            const int R0 = 2 * (warp & 1);
            const bool first = lane < 16;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float x0[16], x1[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) x0[e] = x1[e] = 0.f;
                if (j <= R0) tmem_ld16(tl + TM_G1 + kda_sec(R0) + 16 * j, x0);  // warp-uniform conditions
                if (j <= R0 + 1) tmem_ld16(tl + TM_G1 + kda_sec(R0 + 1) + 16 * j, x1);
                wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) g1[16 * j + e] = first ? x0[e] : x1[e];
            }
            if (a.kwide[ci]) {  // exact in-block entries (row r's own block, columns b(r) .. b(r) + 15)
                const int r = trow & 63, R = r >> 4;
                const float *dx = a.Dx + (((size_t)ci * 2 + (trow < 64 ? 0 : 1)) * C + r) * 16;
                float d[16];
#pragma unroll
                for (int e = 0; e < 16; e += 4) {
                    const float4 t4 = *reinterpret_cast<const float4 *>(dx + e);
                    d[e] = t4.x; d[e + 1] = t4.y; d[e + 2] = t4.z; d[e + 3] = t4.w;
                }
#pragma unroll
                for (int i = 0; i < 64; ++i)
                    if ((i >> 4) == R) g1[i] = d[i & 15];
            }
        } else {
            tmem_row64(tl + TM_G1, g1);
        }
        const bool big = *bigflag != 0;
        const float *gc = pf + PF_GC * 64, *cola = pf + PF_COLA * 64;
        const bool arow = trow < 64;
        const int r = arow ? trow : trow - 64;
        // gate factor of each (r, i): e^{g_r - g_i}, split at the midpoint unless the range is large
        float f[64];
        if (VAR != VAR_GATED) {  // DeltaNet; KDA carries its gates in the operands
#pragma unroll
            for (int i = 0; i < 64; ++i) f[i] = 1.f;
        } else if (!big) {
            const float rf = pf[PF_ROWP * 64 + r];
#pragma unroll
            for (int i4 = 0; i4 < 16; ++i4) {
                const float4 c = reinterpret_cast<const float4 *>(cola)[i4];
                f[4 * i4] = c.x * rf; f[4 * i4 + 1] = c.y * rf; f[4 * i4 + 2] = c.z * rf; f[4 * i4 + 3] = c.w * rf;
            }
        } else {
            const float gr = gc[r];
#pragma unroll
            for (int i = 0; i < 64; ++i) f[i] = (i <= r) ? __expf(gr - gc[i]) : 0.f;
        }
        if (RAW) {  // the raw rows' norms: row factor 1/|k_r| or 1/|q_r|, column factor 1/|k_i|
            const float rr = pf[(arow ? PF_RNK : PF_RNQ) * 64 + r];
            const float *rk = pf + PF_RNK * 64;
#pragma unroll
            for (int i = 0; i < 64; ++i) f[i] *= rr * rk[i];
        }
        if (arow) {
            // k k^T row (KEEP) into the q_p0 tile, free since P1 completed
            if (KEEP) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) st_chunk(sm + OFF_KQ + 8192, swz(r, ch), g1 + ch * 8);
            }
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
        } else {
#pragma unroll
            for (int i = 0; i < 64; ++i) g1[i] = (i <= r) ? g1[i] * f[i] : 0.f;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) st_chunk(sm + OFF_P, swz(r, ch), g1 + ch * 8);
        }
    }
    fence_proxy_async();
    fence_before_sync();
    ok = consensus(ok);
    if (ok && tid == 0) {
        fence_after_sync();
        tma_store_2d(&mp.P, sm + OFF_P, 0, ci * C);
        if (KEEP) tma_store_2d(&mp.KK, sm + OFF_KQ + 8192, 0, ci * C);
        bulk_commit();
    }
    // ---------------- T = (I + A)^-1 ----------------
    float *ysc = reinterpret_cast<float *>(sm + OFF_KQ + 24576);  // q_p1, free after P1
    if (ok) unit_lower_inverse64(Asc, Tf, ysc, tid, sync);
    // ---------------- T diag(beta), T diag(beta e^g) tiles; T itself (KEEP) ----------------
    if (KEEP) {  // the P and k k^T stores have read the tiles that T and T diag(beta) take over
        if (tid == 0) bulk_wait_read_all();
        sync();
    }
    if (ok) {
        const int i = tid & 63;
        const float *fac = pf + (tid < 64 ? PF_BV : PF_BK) * 64;
        unsigned char *dst = sm + OFF_KQ + (tid < 64 ? 8192 : 24576);
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
            const float4 lo = *reinterpret_cast<const float4 *>(&Tf[sw64(i, ch * 8)]);
            const float4 hi = *reinterpret_cast<const float4 *>(&Tf[sw64(i, ch * 8 + 4)]);
            float w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) w[e] = (ch * 8 + e <= i) ? w[e] : 0.f;
            if (KEEP && tid < 64) st_chunk(sm + OFF_P, swz(i, ch), w);
#pragma unroll
            for (int e = 0; e < 8; ++e) w[e] *= fac[ch * 8 + e];
            if (RAW && tid >= 64) {  // W's operand k is the normalised one: 1/|k_j| per column
#pragma unroll
                for (int e = 0; e < 8; ++e) w[e] *= pf[PF_RNK * 64 + ch * 8 + e];
            }
            st_chunk(dst, swz(i, ch), w);
        }
    }
    fence_proxy_async();
    fence_before_sync();
    ok = consensus(ok);
    // ---------------- W = [T diag(beta e^g) ; *] k,  U~ = [T diag(beta) ; *] v ----------------
    if (ok && tid == 0) {
        fence_after_sync();
        if (KEEP) {
            tma_store_2d(&mp.Tn, sm + OFF_P, 0, ci * C);
            bulk_commit();
        }
        const uint32_t id = idesc_bf16(128, 128, 0, 1);
        const uint64_t dkb = VAR == VAR_KDA ? sdesc(smem_u32(sm + OFF_X), 8192, 1024) : sdesc(skq, 16384, 1024);
#pragma unroll
        for (int st = 0; st < 4; ++st) {
            mma_bf16(tbase + TM_XW, sdesc(skq + 24576 + st * 32, 16, 1024), sdesc_at(dkb, st * 2048), id, st > 0);
            mma_bf16(tbase + TM_XU, sdesc(skq + 8192 + st * 32, 16, 1024), sdesc(sv + st * 2048, 8192, 1024), id,
                     st > 0);
        }
        mma_commit(&bar[1]);
        mma_issued++;
    }
    if (ok) ok = consensus(wait_mma());
    if (ok && trow < 64) {
        const int r = trow;
#pragma unroll
        for (int x = 0; x < 4; ++x) {  // W panels 0, 1, then U~ panels 0, 1
            float v[64];
            tmem_row64(tl + (x < 2 ? TM_XW : TM_XU) + (x & 1) * 64, v);
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) st_chunk(sm + OFF_F, (uint32_t)x * 8192 + swz(r, ch), v + ch * 8);
        }
    }
    fence_proxy_async();
    fence_before_sync();
    ok = consensus(ok);
    if (tid == 0) {
        if (ok) {
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                tma_store_2d(&mp.W, sm + OFF_F + p * 8192, 64 * p, ci * C);
                tma_store_2d(&mp.Ut, sm + OFF_F + 16384 + p * 8192, 64 * p, ci * C);
            }
            bulk_commit();
        }
        bulk_wait_all();
        if (*abort_flag) {  // let whatever was issued finish before the CTA leaves
            volatile int dummy = 0;
            mbar_wait(&bar[0], 0, &dummy, 100000000ull);
            if (mma_issued > 0) mbar_wait(&bar[1], (mma_issued - 1) & 1, &dummy, 100000000ull);
        }
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == 0) tmem_dealloc(tbase, TM_COLS);
}

// ---------------------------------------------------------------- KDA gate operands
// One CTA of 128 threads per chunk.  Thread (tg, cg) = (tid / 16, tid % 16) owns key channels
// 8 cg ... 8 cg + 7 of tokens 8 tg ... 8 tg + 7, so every access moves 16 bytes; warp w holds
// the 16 tokens of block w.  The in-chunk cumulative log gate g of each channel is a prefix sum
// over the chunk's tokens (tokens past T add nothing): inside the thread's 8 tokens, then across
// the 8 token groups through shared memory.  Then every gate-scaled operand the split path needs
// is written row-major per chunk.  The factors e^{g_r - g_b(r)}, e^{g}, e^{g_C - g} and the column
// factors of earlier tokens are <= 1 (log alpha <= 0); only the in-block column factors grow,
// and their exponent is clamped at 80 (chunks where it would pass KDA_DIAG_SPAN are marked).
struct KdaArgs {
    const __nv_bfloat16 *q, *k, *alpha;
    __nv_bfloat16 *Kt1, *Qt1, *Kh, *Kt, *Qt, *Kb;
    float *egc;
    int *kwide;
    float *Dx;
    float *G;  // optional: g itself, fp32 [chunks][64][128] (written for the marked chunks only)
    int T, H, N;
    int n0;    // chunk of blockIdx.x = 0 (a launch may cover chunks n0 ..)
};

__device__ __forceinline__ void unpack8_bf16(const uint4 x, float *v) {
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ void st8_bf16(__nv_bfloat16 *p, const float *v) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = pack_bf16(v[2 * i], v[2 * i + 1]);
    *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

// shared memory of k_kda_gates: g [64][128] fp32, k and q [64][128] bf16, block sums and edges
constexpr uint32_t KG_G = 0, KG_K = 32768, KG_Q = 49152, KG_TOT = 65536, KG_BLK = KG_TOT + 8 * DK * 4,
                   KG_END = KG_BLK + 4 * DK * 4, KG_SMEM = KG_END + DK * 4;

// 16 bytes global -> shared without registers (zeros when !in)
__device__ __forceinline__ void cp16(void *dst, const void *src, bool in) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(in ? 16 : 0)
                 : "memory");
}

__global__ void __launch_bounds__(128) k_kda_gates(KdaArgs a) {
    extern __shared__ __align__(16) unsigned char kg_sm[];
    float *sg = reinterpret_cast<float *>(kg_sm + KG_G);
    __nv_bfloat16 *sk = reinterpret_cast<__nv_bfloat16 *>(kg_sm + KG_K), *sq = reinterpret_cast<__nv_bfloat16 *>(kg_sm + KG_Q);
    float(*tot)[DK] = reinterpret_cast<float(*)[DK]>(kg_sm + KG_TOT);
    float(*gblk)[DK] = reinterpret_cast<float(*)[DK]>(kg_sm + KG_BLK);
    float *gend = reinterpret_cast<float *>(kg_sm + KG_END);
    const int n = a.n0 + (int)blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tg = threadIdx.x >> 4, cg = threadIdx.x & 15, c0 = 8 * cg, R = tg >> 1;
    const int t0 = n * C, L = min(C, a.T - t0);
    const size_t ci = ((size_t)b * a.H + h) * a.N + n;
    auto at = [&](int r) { return (((size_t)b * a.T + t0 + r) * a.H + h) * DK + c0; };
    // every input row of this thread at once: k and q straight into shared memory, log alpha into
    // registers (24 16-byte loads in flight; rows past T read as 0)
    uint4 ar[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int tr = 8 * tg + r;
        const bool in = tr < L;
        const size_t src = in ? at(tr) : 0;
        cp16(sk + tr * DK + c0, a.k + src, in);
        cp16(sq + tr * DK + c0, a.q + src, in);
        ar[r] = in ? __ldg(reinterpret_cast<const uint4 *>(a.alpha + src)) : make_uint4(0u, 0u, 0u, 0u);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    float g[8][8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        float x[8];
        unpack8_bf16(ar[r], x);
#pragma unroll
        for (int j = 0; j < 8; ++j) g[r][j] = (r ? g[r - 1][j] : 0.f) + x[j];
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) tot[tg][c0 + j] = g[7][j];
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float off = 0.f;
        for (int t2 = 0; t2 < tg; ++t2) off += tot[t2][c0 + j];
#pragma unroll
        for (int r = 0; r < 8; ++r) g[r][j] += off;
        if ((tg & 1) == 0) gblk[R][c0 + j] = g[0][j];  // token 16 R, the first of block R
        if (tg == 7) gend[c0 + j] = g[7][j];           // token C - 1, the last
    }
    // this thread's g rows to shared memory (read back row by row below)
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        float *d = sg + (8 * tg + r) * DK + c0;
        *reinterpret_cast<float4 *>(d) = make_float4(g[r][0], g[r][1], g[r][2], g[r][3]);
        *reinterpret_cast<float4 *>(d + 4) = make_float4(g[r][4], g[r][5], g[r][6], g[r][7]);
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    float gb[8], gC[8];  // g at the first token of this thread's block, and at the chunk's last
    bool wide = false;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        gb[j] = gblk[R][c0 + j];
        gC[j] = gend[c0 + j];
        // the fall of the gate inside block R, from its first token to its last (held by tg odd)
        if (tg & 1) wide |= !(gb[j] - g[7][j] <= KDA_DIAG_SPAN);
    }
#pragma unroll 1
    for (int r = 0; r < 8; ++r) {
        const int tr = 8 * tg + r;
        float kr[8], qr[8], gr[8];
        unpack8_bf16(*reinterpret_cast<const uint4 *>(sk + tr * DK + c0), kr);
        unpack8_bf16(*reinterpret_cast<const uint4 *>(sq + tr * DK + c0), qr);
        {
            const float4 u0 = *reinterpret_cast<const float4 *>(sg + tr * DK + c0);
            const float4 u1 = *reinterpret_cast<const float4 *>(sg + tr * DK + c0 + 4);
            gr[0] = u0.x; gr[1] = u0.y; gr[2] = u0.z; gr[3] = u0.w;
            gr[4] = u1.x; gr[5] = u1.y; gr[6] = u1.z; gr[7] = u1.w;
        }
        float o1[8], o2[8], o4[8], o5[8], o6[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            // every exponent here is <= 0 for log alpha <= 0; the clamp only keeps other input finite
            const float eb = __expf(fminf(gr[j] - gb[j], 80.f));  // row factor
            const float eg = __expf(fminf(gr[j], 80.f)), ec = __expf(fminf(gC[j] - gr[j], 80.f));
            o1[j] = kr[j] * eb; o2[j] = qr[j] * eb;
            o4[j] = kr[j] * eg; o5[j] = qr[j] * eg; o6[j] = kr[j] * ec;
        }
        const size_t o = (ci * C + tr) * DK + c0;
        st8_bf16(a.Kt1 + o, o1);
        st8_bf16(a.Qt1 + o, o2);
        st8_bf16(a.Kt + o, o4);
        st8_bf16(a.Qt + o, o5);
        st8_bf16(a.Kb + o, o6);
        // column operand of every block R2 >= R (token tr is one of its rows 0 .. 16 R2 + 15)
#pragma unroll 1
        for (int R2 = R; R2 < 4; ++R2) {
            float oh[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) oh[j] = kr[j] * __expf(fminf(gblk[R2][c0 + j] - gr[j], 80.f));
            st8_bf16(a.Kh + (ci * KDA_KH_ROWS + kda_sec(R2) + tr) * DK + c0, oh);
        }
    }
    if (tg == 0) {
        float e[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) e[j] = __expf(fminf(gC[j], 80.f));
        *reinterpret_cast<float4 *>(a.egc + ci * DK + c0) = make_float4(e[0], e[1], e[2], e[3]);
        *reinterpret_cast<float4 *>(a.egc + ci * DK + c0 + 4) = make_float4(e[4], e[5], e[6], e[7]);
    }
    wide = __syncthreads_or(wide);
    if (threadIdx.x == 0) a.kwide[ci] = wide ? 1 : 0;
    if (wide && a.G) {  // g itself, for the CUDA-core gradient kernel that takes the marked chunks
#pragma unroll 1
        for (int r = 0; r < 8; ++r) {
            const float *src = sg + (8 * tg + r) * DK + c0;
            float *dst = a.G + (ci * C + 8 * tg + r) * DK + c0;
            *reinterpret_cast<float4 *>(dst) = *reinterpret_cast<const float4 *>(src);
            *reinterpret_cast<float4 *>(dst + 4) = *reinterpret_cast<const float4 *>(src + 4);
        }
    }
}

// The exact in-block sums of the chunks k_kda_gates marked (one CTA of 128 threads per chunk;
// the others return at once).  Thread c forms channel c's cumulative log gate; then warp w takes
// the pairs i <= r of block w, lane l channels l, l + 32, l + 64, l + 96, with one exponential
// per pair and channel (every exponent <= 0):
//   Dx[0][r][i - 16 w] = sum_c k_rc k_ic e^{g_rc - g_ic},  Dx[1][r][i - 16 w] = sum_c q_rc k_ic e^{g_rc - g_ic}
// (0 for i > r).  smem: g, k, q [64][128] fp32.
constexpr uint32_t DIAG_SMEM = 3 * C * DK * 4;

__global__ void __launch_bounds__(128) k_kda_diag(KdaArgs a) {
    const int n = a.n0 + (int)blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const size_t ci = ((size_t)b * a.H + h) * a.N + n;
    if (!a.kwide[ci]) return;  // uniform over the CTA
    extern __shared__ float dsm[];
    float *gsm = dsm, *ksm = gsm + C * DK, *qsm = ksm + C * DK;
    const int t0 = n * C, L = min(C, a.T - t0), c = threadIdx.x, warp = c >> 5, lane = c & 31;
    float run = 0.f;
    for (int r = 0; r < C; ++r) {
        float kv = 0.f, qv = 0.f;
        if (r < L) {
            const size_t x = (((size_t)b * a.T + t0 + r) * a.H + h) * DK + c;
            run += __bfloat162float(a.alpha[x]);
            kv = __bfloat162float(a.k[x]);
            qv = __bfloat162float(a.q[x]);
        }
        gsm[r * DK + c] = run;
        ksm[r * DK + c] = kv;
        qsm[r * DK + c] = qv;
    }
    __syncthreads();
    const int r0 = 16 * warp;
    for (int r = r0; r < r0 + 16; ++r) {
        for (int i = r0; i < r0 + 16; ++i) {
            float sk = 0.f, sq = 0.f;
            if (i <= r) {
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int cc = lane + 32 * m;
                    const float e = __expf(gsm[r * DK + cc] - gsm[i * DK + cc]) * ksm[i * DK + cc];
                    sk += ksm[r * DK + cc] * e;
                    sq += qsm[r * DK + cc] * e;
                }
                sk = warp_sum(sk);
                sq = warp_sum(sq);
            }
            if (lane == 0) {
                a.Dx[((ci * 2 + 0) * C + r) * 16 + (i - r0)] = sk;
                a.Dx[((ci * 2 + 1) * C + r) * 16 + (i - r0)] = sq;
            }
        }
    }
}

template <int VAR, int KEEP, int RAW = 0>
static cudaError_t launch_prep(const Maps &mp, const Args &a, dim3 grid, cudaStream_t s, Rec &rec) {
    const size_t smem = (VAR == VAR_KDA ? SMEM_KDA : SMEM_BYTES) + 1024;
    cudaError_t e =
        cudaFuncSetAttribute(k_chunk_prep<VAR, KEEP, RAW>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    rec.mark(s);
    k_chunk_prep<VAR, KEEP, RAW><<<grid, NTHREADS, smem, s>>>(mp, a);
    return cudaGetLastError();
}

}  // namespace tcp

cudaError_t tc_kda_gates(const Geo &g, const Tensors &t, const TcWs &w, float *G, cudaStream_t s, Rec &rec) {
    using namespace tcp;
    KdaArgs a;
    a.q = (const __nv_bfloat16 *)t.q; a.k = (const __nv_bfloat16 *)t.k; a.alpha = (const __nv_bfloat16 *)t.alpha;
    a.Kt1 = w.Kt1; a.Qt1 = w.Qt1; a.Kh = w.Kh; a.Kt = w.Kt; a.Qt = w.Qt; a.Kb = w.Kb; a.egc = w.egc; a.G = G;
    a.kwide = w.kwide; a.Dx = w.Dx;
    a.T = g.T; a.H = g.H; a.N = g.N;
    a.n0 = w.m0;  // the chunks [m0, m1) of each sequence (m1 = 0: to the end)
    const unsigned ns = (unsigned)((w.m1 > 0 ? w.m1 : g.N) - w.m0);
    cudaError_t e = cudaFuncSetAttribute(k_kda_diag, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)DIAG_SMEM);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(k_kda_gates, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)KG_SMEM);
    if (e != cudaSuccess) return e;
    rec.mark(s);
    k_kda_gates<<<dim3(ns, g.H, g.B), DK, KG_SMEM, s>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    rec.mark(s);
    k_kda_diag<<<dim3(ns, g.H, g.B), DK, DIAG_SMEM, s>>>(a);
    return cudaGetLastError();
}

namespace tcp {
// bf16 -> fp32 copies of up to five arrays (8 elements a thread, grid-stride)
struct Widen {
    const __nv_bfloat16 *src[5];
    float *dst[5];
    size_t n8[5];     // elements / 8
    size_t per8[5];   // elements / 8 of one chunk
    const int *only;  // optional: widen the chunks flagged here alone
};
__global__ void __launch_bounds__(256) k_widen(Widen a) {
    for (int i = 0; i < 5; ++i) {
        if (!a.src[i]) continue;
        for (size_t x = (size_t)blockIdx.x * 256 + threadIdx.x; x < a.n8[i]; x += (size_t)gridDim.x * 256) {
            if (a.only && !a.only[x / a.per8[i]]) continue;
            const uint4 v = reinterpret_cast<const uint4 *>(a.src[i])[x];
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
            float f[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                f[2 * j] = __uint_as_float(w4[j] << 16);
                f[2 * j + 1] = __uint_as_float(w4[j] & 0xFFFF0000u);
            }
            float4 *d = reinterpret_cast<float4 *>(a.dst[i] + 8 * x);
            d[0] = make_float4(f[0], f[1], f[2], f[3]);
            d[1] = make_float4(f[4], f[5], f[6], f[7]);
        }
    }
}
}  // namespace tcp

cudaError_t tc_to_simt(const Geo &g, const TcWs &w, float *W, float *Ut, float *P, float *Sn, float *Un, cudaStream_t s,
                       Rec &rec, const int *only) {
    using namespace tcp;
    const size_t nc = (size_t)g.B * g.H * g.N;
    Widen a = {};
    const __nv_bfloat16 *src[5] = {w.W, w.Ut, w.P, w.Sn, w.Un};
    float *dst[5] = {W, Ut, P, Sn, Un};
    const size_t per[5] = {(size_t)C * DK, (size_t)C * DV, (size_t)C * C, (size_t)DK * DV, (size_t)C * DV};
    for (int i = 0; i < 5; ++i) {  // an absent destination is not widened
        a.src[i] = dst[i] ? src[i] : nullptr;
        a.dst[i] = dst[i];
        a.n8[i] = nc * per[i] / 8;
        a.per8[i] = per[i] / 8;
    }
    a.only = only;
    rec.mark(s);
    k_widen<<<148 * 8, 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t tc_rev_to_simt(const Geo &g, const TcWs &w, float *dSn, float *dUn, cudaStream_t s, Rec &rec,
                           const int *only) {
    using namespace tcp;
    const size_t nc = (size_t)g.B * g.H * g.N;
    Widen a = {};
    a.src[0] = dSn ? w.dSn : nullptr; a.dst[0] = dSn; a.n8[0] = nc * DK * DV / 8; a.per8[0] = DK * DV / 8;
    a.src[1] = dUn ? w.dUn : nullptr; a.dst[1] = dUn; a.n8[1] = nc * C * DV / 8; a.per8[1] = C * DV / 8;
    a.only = only;
    rec.mark(s);
    k_widen<<<148 * 8, 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t tc_chunk_prep(const Geo &g, const Tensors &t, const TcWs &w, bool keep, cudaStream_t s, Rec &rec,
                          bool raw) {
    using namespace tcp;
    Maps mp;
    const uint64_t Bn = g.B, T = g.T, H = g.H, NC = (uint64_t)g.B * g.H * g.N;
    bool ok = tc::make_map_4d_bf16(&mp.q, t.q, DK, H, T, Bn, 64) && tc::make_map_4d_bf16(&mp.k, t.k, DK, H, T, Bn, 64) &&
              tc::make_map_4d_bf16(&mp.v, t.v, DV, H, T, Bn, 64) && tc::make_map_2d_bf16(&mp.W, w.W, DK, NC * C, 64) &&
              tc::make_map_2d_bf16(&mp.Ut, w.Ut, DV, NC * C, 64) && tc::make_map_2d_bf16(&mp.P, w.P, C, NC * C, 64);
    if (ok && keep)
        ok = tc::make_map_2d_bf16(&mp.KK, w.KK, C, NC * C, 64) && tc::make_map_2d_bf16(&mp.Tn, w.Tn, C, NC * C, 64);
    if (ok && g.variant == VAR_KDA)
        ok = tc::make_map_2d_bf16(&mp.Kt1, w.Kt1, DK, NC * C, 64) && tc::make_map_2d_bf16(&mp.Qt1, w.Qt1, DK, NC * C, 64) &&
             tc::make_map_2d_bf16(&mp.Kh, w.Kh, DK, NC * KDA_KH_ROWS, KDA_KH_ROWS) &&
             tc::make_map_2d_bf16(&mp.Kt, w.Kt, DK, NC * C, 64);
    if (!ok) return cudaErrorInvalidValue;
    Args a;
    a.alpha = t.alpha; a.beta = t.beta; a.gb = w.gb; a.kwide = w.kwide; a.Dx = w.Dx; a.rn = w.rn;
    a.B = g.B; a.T = g.T; a.H = g.H; a.N = g.N;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return cudaErrorInvalidValue;
    a.wave = 2 * sms;
    a.n0 = w.m0;  // the chunks [m0, m1) of each sequence (m1 = 0: to the end)
    const dim3 grid((w.m1 > 0 ? w.m1 : g.N) - w.m0, g.H, g.B);
    if (g.variant == VAR_KDA) {  // KEEP: T and the gated k k^T products M (for the KDA gradient kernel)
        if (raw) return cudaErrorInvalidValue;
        return keep ? launch_prep<VAR_KDA, 1>(mp, a, grid, s, rec) : launch_prep<VAR_KDA, 0>(mp, a, grid, s, rec);
    }
    if (raw) {
        if (keep || !w.rn) return cudaErrorInvalidValue;
        return g.variant == VAR_GATED ? launch_prep<VAR_GATED, 0, 1>(mp, a, grid, s, rec)
                                      : launch_prep<VAR_DELTANET, 0, 1>(mp, a, grid, s, rec);
    }
    if (g.variant == VAR_GATED)
        return keep ? launch_prep<VAR_GATED, 1>(mp, a, grid, s, rec) : launch_prep<VAR_GATED, 0>(mp, a, grid, s, rec);
    return keep ? launch_prep<VAR_DELTANET, 1>(mp, a, grid, s, rec) : launch_prep<VAR_DELTANET, 0>(mp, a, grid, s, rec);
}

}  // namespace dr
