// clvr.cu -- cross-layer value routing: h_out = h + U W and its gradients.
//
// ETH news page on the architecture study, section 七 (and the explainer's CLVR section): a
// layer's write values u_t = beta_t (v_t - S'_t^T k_t) enter a higher layer's hidden stream, the
// residual stream all layers share, through a projection W that starts at zero.  With U the write
// values as [B*T, H*dv] (the core's u output, unchanged), W [H*dv, D] and h [B*T, D]:
//     h_out = h + U W,      dU = dH W^T,      dW = U^T dH,      dh = dH.
//
// bf16: one persistent tcgen05 GEMM kernel serves all three products.  Its CTAs come in pairs
// (2-CTA clusters) that compute 256 x 256 output tiles together with cta_group::2 MMAs
// (M = 256, N = 256): each CTA of a pair holds 128 rows of the A slice and 128 columns of the B
// slice, and the tensor cores of the two SMs share their B halves, so that each SM loads and
// reads 32 KB of operands per 64-wide K slice instead of the 48 KB a one-SM 128 x 256 tile needs.
// In each CTA warp 0 feeds a five-stage ring of K slices by TMA (the loads of both CTAs complete
// on the first CTA's barrier), warp 1 of the first CTA issues the MMAs (fp32 accumulators in
// TMEM, each CTA holding its 128 rows; two accumulators, so that a tile's epilogue overlaps the
// next tile's products), warps 2-5 of each CTA drain its rows.  Either operand may be stored
// K-major or MN-major (U^T and W^T are read in place, no transposes):
//   h_out = h + U W     A = U K-major,    B = W MN-major,   residual tile h added in the epilogue
//   dU    = dH W^T      A = dH K-major,   B = W K-major
//   dW    = U^T dH      A = U MN-major,   B = dH MN-major,  fp32 out; the long reduction over the
//                       tokens is split into slices whose fp32 partials a second kernel adds in a
//                       fixed order (deterministic)
// The bf16 results leave through TMA stores of the output tile, rows and columns past the matrix
// clipped; loads past it read zeros.  fp32 I/O runs a register-blocked CUDA-core GEMM in fp32.
#include "../../include/delta_rule.h"
#include "clvr.cuh"
#include "tc_host.cuh"
#include "tc_ptx.cuh"
#include "tc_tile.cuh"

namespace dr {
namespace clv {

using namespace dr::tc;
using dr::tcf::ld_chunk;
using dr::tcf::st_chunk;

constexpr int BM = 256, BN = 256, BK = 64, STAGES = 5;  // a CTA pair's output tile, K slice, ring depth
constexpr int HM = BM / 2, HN = BN / 2;                 // one CTA's rows of A and D, its columns of B
constexpr uint32_t A_BYTES = HM * BK * 2, B_BYTES = HN * BK * 2;  // 16 KB, 16 KB per stage and CTA
constexpr uint32_t OFF_A = 0, OFF_B = STAGES * A_BYTES, OFF_C = OFF_B + STAGES * B_BYTES;
constexpr uint32_t C_BYTES = HM * BN * 2;  // this CTA's bf16 output rows: 4 panels [128 rows][64 columns]
constexpr uint32_t OFF_MISC = OFF_C + C_BYTES;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 256;
// FULL (first CTA only): both CTAs' loads of a stage have landed; EMPTY: the MMAs have read a
// stage; ACCF: an accumulator is complete; ACCE (first CTA only): the 8 epilogue warps of the pair
// have drained an accumulator; B_CF + p: panel p (64 columns) of a tile's residual has landed
enum { B_FULL = 0, B_EMPTY = STAGES, B_ACCF = 2 * STAGES, B_ACCE = B_ACCF + 2, B_CF = B_ACCE + 2, B_NUM = B_CF + 4 };
constexpr uint32_t M_TMEM = 8 * B_NUM, M_ABORT = M_TMEM + 4;
static_assert(M_ABORT + 4 <= 256, "misc overflow");
static_assert(SMEM_BYTES + 1024 <= 232448, "shared memory");
constexpr int NTHREADS = 192;  // warp 0 TMA, warp 1 MMA and TMEM owner, warps 2-5 epilogue
constexpr uint32_t TM_COLS = 512;  // two 256-column accumulators
constexpr int MAX_SPLIT = 8;
constexpr size_t WS = (size_t)32 << 20;  // split-reduction partials of dW (fp32)

struct Maps {
    CUtensorMap a, b;  // operands (box per layout below)
    CUtensorMap c, d;  // bf16 residual and output [M][N], box 64 columns x 128 rows
};

struct Args {
    int M, N, K;      // D [M][N] = op(A) [M][K] op(B) [K][N]
    int a_mn, b_mn;   // 1: the operand is stored MN-major (its K index is the row)
    int has_c;        // add the residual tile of map c
    float *d32;       // fp32 output (slice s at d32 + s * slice_elems) instead of the bf16 map d
    size_t slice_elems;
    int nsplit, kslice;  // slice s reduces k in [s kslice, min(K, (s + 1) kslice)), kslice % 64 == 0
};

// at most N of this thread's committed bulk groups still reading shared memory (N a constant 0..7)
template <int N>
__device__ __forceinline__ void bulk_wait_read_n() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Shared-memory descriptor of K step kk (16 elements) of an operand tile laid out as above
__device__ __forceinline__ uint64_t operand_desc(uint32_t base, bool mn, int kk) {
    return mn ? sdesc(base + kk * 2048, 8192, 1024) : sdesc(base + kk * 32, 16, 1024);
}

// ---- the CTA-pair forms (every tcgen05 instruction of the kernel names cta_group::2)
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// one warp of each CTA of the pair takes part; both receive the same column address
__device__ __forceinline__ void tmem_alloc_pair(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D (256 rows: 128 in each CTA's TMEM) += A (128 rows from each CTA) B (N / 2 columns from each CTA)
__device__ __forceinline__ void mma_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, int accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
}
// one arrival on the mbarrier at a shared::cluster address (this CTA's or the peer's) once this
// thread's MMAs so far are complete
__device__ __forceinline__ void commit_pair(uint32_t bar_cluster) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_cluster)
                 : "memory");
}
// 2-D tiled load into this CTA's shared memory, completion counted on an mbarrier of either CTA
__device__ __forceinline__ void tma_load_pair(void *dst, const CUtensorMap *map, int c0, int c1, uint32_t bar_cluster) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
        "%3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar_cluster)
        : "memory");
}
__device__ __forceinline__ void arrive_remote(uint32_t bar_cluster) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}
// bounded wait (as mbar_wait) with cluster-scope acquire: the phase may be completed by the peer
__device__ __forceinline__ bool mbar_wait_pair(uint64_t *bar, uint32_t parity, volatile int *abort,
                                               uint64_t limit_ns = 1000000000ull) {
    auto try_once = [&]() -> bool {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(ok)
            : "r"(smem_u32(bar)), "r"(parity)
            : "memory");
        return ok != 0;
    };
    if (try_once()) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (try_once()) return true;
        if ((it & 63) == 0) {
            if (*abort) return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                atomicOr(&g_dev_error, DEVERR_TIMEOUT);
                *abort = 1;
                return false;
            }
        }
    }
}

// Loads of one K slice of one operand tile into this CTA's shared memory (the layouts the MMA
// reads), completion counted on the first CTA's barrier (shared::cluster address):
//   K-major, R rows: one box of 64 (K) x R rows -> [R rows][128 B], 128-byte swizzle
//   MN-major, R columns: R / 64 boxes of 64 (MN) x 64 (K rows) -> panel p = [64 K rows][128 B]
__device__ __forceinline__ void load_operand(unsigned char *dst, const CUtensorMap *map, bool mn, int rows, int r0,
                                             int k0, uint32_t bar_cluster) {
    if (!mn) {
        tma_load_pair(dst, map, k0, r0, bar_cluster);
    } else {
        for (int p = 0; p < rows / 64; ++p) tma_load_pair(dst + p * 8192, map, r0 + 64 * p, k0, bar_cluster);
    }
}

__global__ void __launch_bounds__(NTHREADS, 1) k_gemm_tc(const __grid_constant__ Maps mp, Args a) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + OFF_MISC);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC + M_TMEM);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + OFF_MISC + M_ABORT);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();  // 0: the CTA that issues the MMAs
    const bool lead = rank == 0;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int mt = (a.M + BM - 1) / BM, nt = (a.N + BN - 1) / BN;
    const int tiles = mt * nt * a.nsplit;
    const int kblocks_full = (a.kslice + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int i = 0; i < B_NUM; ++i) mbar_init(&bar[i], (i >= B_ACCE && i < B_CF) ? 8 : 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc_pair(tmem_slot, TM_COLS);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    cluster_sync();  // both CTAs' barriers are initialised before any copy or arrival reaches them
    const uint32_t tbase = *tmem_slot;
    // barrier i of the first CTA / of the second, as shared::cluster addresses
    auto lead_bar = [&](int i) { return map_to_rank(&bar[i], 0); };
    auto peer_bar = [&](int i) { return map_to_rank(&bar[i], 1); };

    // tile t -> split slice, row block, column block (consecutive tiles share the A rows)
    auto tile_of = [&](int t, int &s, int &mb, int &nb) {
        s = t % a.nsplit;
        const int r = t / a.nsplit;
        nb = r % nt;
        mb = r / nt;
    };
    auto kblocks_of = [&](int s) {
        const int k0 = s * a.kslice, k1 = min(a.K, k0 + a.kslice);
        return k1 > k0 ? min(kblocks_full, (k1 - k0 + BK - 1) / BK) : 0;
    };

    if (warp == 0) {
        // ================================ TMA producer ================================
        // both CTAs: this CTA's 128 rows of the A slice and 128 columns of the B slice; the first
        // CTA's FULL barrier expects the bytes of both
        int slot = 0, use = 0, nissued = 0;
        for (int t = pair; t < tiles; t += npairs) {
            int s, mb, nb;
            tile_of(t, s, mb, nb);
            const int nk = kblocks_of(s);
            for (int kb = 0; kb < nk; ++kb) {
                if (use > 0 && !mbar_wait_pair(&bar[B_EMPTY + slot], (use - 1) & 1, abort_flag)) goto producer_done;
                if (lane == 0) {
                    const int k0 = s * a.kslice + kb * BK;
                    const uint32_t full = lead_bar(B_FULL + slot);
                    if (lead) mbar_arrive_tx(&bar[B_FULL + slot], 2 * (A_BYTES + B_BYTES));
                    load_operand(sm + OFF_A + slot * A_BYTES, &mp.a, a.a_mn, HM, mb * BM + HM * (int)rank, k0, full);
                    load_operand(sm + OFF_B + slot * B_BYTES, &mp.b, a.b_mn, HN, nb * BN + HN * (int)rank, k0, full);
                }
                __syncwarp();
                ++nissued;
                if (++slot == STAGES) { slot = 0; ++use; }
            }
        }
    producer_done:
        if (*abort_flag && lane == 0) {  // let the issued copies land before the CTA retires
            if (lead) {  // the stages' phases count both CTAs' bytes
                volatile int dummy = 0;
                for (int i = 0; i < STAGES; ++i) {  // stage i was filled nissued / STAGES (+1) times
                    const int uses = nissued / STAGES + (i < nissued % STAGES ? 1 : 0);
                    if (uses > 0) mbar_wait(&bar[B_FULL + i], (uses - 1) & 1, &dummy, 100000000ull);
                }
            } else {  // this CTA's copies complete on the first CTA's barriers: give them 1 ms
                const uint64_t t0 = globaltimer_ns();
                while (globaltimer_ns() - t0 < 1000000ull) {
                }
            }
        }
    } else if (warp == 1) {
        // ================================ MMA issuer ================================
        // first CTA only (the second CTA's warp 1 only shares the TMEM allocation)
        const uint32_t id = idesc_bf16(BM, BN, a.a_mn, a.b_mn);
        int slot = 0, use = 0, it = 0, committed[2] = {0, 0};
        bool ok = true;
        for (int t = pair; lead && t < tiles && ok; t += npairs, ++it) {
            int s, mb, nb;
            tile_of(t, s, mb, nb);
            const int nk = kblocks_of(s), acc = it & 1;
            // the pair's epilogues of the tile two back have drained this accumulator
            if (it >= 2 && !(ok = mbar_wait_pair(&bar[B_ACCE + acc], ((it >> 1) - 1) & 1, abort_flag))) break;
            fence_after_sync();
            for (int kb = 0; kb < nk; ++kb) {
                if (!(ok = mbar_wait_pair(&bar[B_FULL + slot], use & 1, abort_flag))) break;
                fence_after_sync();
                if (lane == 0) {
                    const uint32_t sa = smem_u32(sm + OFF_A + slot * A_BYTES), sb = smem_u32(sm + OFF_B + slot * B_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        mma_pair(tbase + acc * BN, operand_desc(sa, a.a_mn, kk), operand_desc(sb, a.b_mn, kk), id,
                                 kb > 0 || kk > 0);
                    // frees the stage in both CTAs once these MMAs have read it
                    commit_pair(lead_bar(B_EMPTY + slot));
                    commit_pair(peer_bar(B_EMPTY + slot));
                }
                __syncwarp();
                if (++slot == STAGES) { slot = 0; ++use; }
            }
            if (!ok) break;
            if (lane == 0) {  // nk == 0: completes at once (zero tile)
                commit_pair(lead_bar(B_ACCF + acc));
                commit_pair(peer_bar(B_ACCF + acc));
            }
            __syncwarp();
            committed[acc]++;
        }
        if (lead && *abort_flag && lane == 0) {  // let issued MMAs finish before TMEM is released
            volatile int dummy = 0;
            for (int i = 0; i < 2; ++i)
                if (committed[i] > 0) mbar_wait(&bar[B_ACCF + i], (committed[i] - 1) & 1, &dummy, 100000000ull);
        }
    } else {
        // ================================ epilogue ================================
        // The output tile is staged as four 64-column panels, each stored (one bulk group per panel)
        // as soon as it is formed.  With a residual, the leader loads the next tile's residual panel
        // p as soon as panel p's store has read the staging tile, so that the load is in flight
        // while this CTA's next accumulator fills.  Each CTA drains its own 128 rows of the pair's tile.
        const int q4 = warp & 3, r = q4 * 32 + lane;  // TMEM lane = output row of the tile
        const uint32_t tl = tbase + ((uint32_t)(q4 * 32) << 16);
        const bool leader = warp == 2 && lane == 0;   // issues the residual loads and the stores
        const bool staged = a.d32 == nullptr, resid = staged && a.has_c;
        auto load_resid_panel = [&](int t, int p) {
            int s2, mb2, nb2;
            tile_of(t, s2, mb2, nb2);
            mbar_arrive_tx(&bar[B_CF + p], 16384);
            tma_load_2d(sm + OFF_C + p * 16384, &mp.c, nb2 * BN + 64 * p, mb2 * BM + HM * (int)rank, &bar[B_CF + p]);
        };
        if (resid && leader && pair < tiles)
            for (int p = 0; p < 4; ++p) load_resid_panel(pair, p);
        int it = 0;
        for (int t = pair; t < tiles; t += npairs, ++it) {
            int s, mb, nb;
            tile_of(t, s, mb, nb);
            const int acc = it & 1;
            const bool zero = kblocks_of(s) == 0;
            bool ok = mbar_wait_pair(&bar[B_ACCF + acc], (it >> 1) & 1, abort_flag);
            fence_after_sync();
            if (named_sync_any(1, 128, !ok || *abort_flag != 0)) break;
            const int row0 = mb * BM + HM * (int)rank, grow = row0 + r;
            bool fail = false;
            for (int p = 0; p < 4; ++p) {
                if (staged) {
                    // the staging panel holds this tile's residual, or is free: the store of the
                    // same panel one tile back has read it (the leader waited before reloading it)
                    bool pok = true;
                    if (resid) pok = mbar_wait(&bar[B_CF + p], (uint32_t)it & 1, abort_flag);
                    else if (leader) bulk_wait_read_n<3>();  // no residual: panel p's previous store is done
                    if (named_sync_any(1, 128, !pok || *abort_flag != 0)) {
                        fail = true;
                        break;
                    }
                }
                float vv[64];  // the panel's 64 columns of this row, one TMEM round trip
#pragma unroll
                for (int q = 0; q < 4; ++q) tmem_ld16(tl + acc * BN + 64 * p + 16 * q, vv + 16 * q);
                wait_ld();
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int c0 = 64 * p + 32 * hh;
                    float *v = vv + 32 * hh;
                    if (zero) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] = 0.f;
                    }
                    if (!staged) {
                        const int gc = nb * BN + c0;
                        if (grow < a.M) {
                            float *dst = a.d32 + (size_t)s * a.slice_elems + (size_t)grow * a.N + gc;
                            if (gc + 32 <= a.N) {
#pragma unroll
                                for (int j = 0; j < 32; j += 4)
                                    *reinterpret_cast<float4 *>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
                            } else {  // static indices keep v in registers
#pragma unroll
                                for (int j = 0; j < 32; ++j)
                                    if (gc + j < a.N) dst[j] = v[j];
                            }
                        }
                    } else {
#pragma unroll
                        for (int ch = 0; ch < 4; ++ch) {
                            const uint32_t o = (uint32_t)p * 16384 + swz(r, ((c0 & 63) >> 3) + ch);
                            if (resid) {
                                float h8[8];
                                ld_chunk(sm + OFF_C, o, h8);
#pragma unroll
                                for (int e = 0; e < 8; ++e) v[ch * 8 + e] += h8[e];
                            }
                            st_chunk(sm + OFF_C, o, v + ch * 8);
                        }
                    }
                }
                if (p == 3) {  // this accumulator is drained (each epilogue warp of the pair arrives once)
                    fence_before_sync();
                    __syncwarp();
                    if (lane == 0) arrive_remote(lead_bar(B_ACCE + acc));
                }
                if (staged) {
                    fence_proxy_async();
                    named_sync(1, 128);
                    if (leader) {
                        tma_store_2d(&mp.d, sm + OFF_C + p * 16384, nb * BN + 64 * p, row0);
                        bulk_commit();
                    }
                }
            }
            if (fail) break;
            // the next tile's residual panels, each once this tile's store of it has read the panel
            if (resid && leader && t + npairs < tiles) {
                bulk_wait_read_n<3>();
                load_resid_panel(t + npairs, 0);
                bulk_wait_read_n<2>();
                load_resid_panel(t + npairs, 1);
                bulk_wait_read_n<1>();
                load_resid_panel(t + npairs, 2);
                bulk_wait_read_n<0>();
                load_resid_panel(t + npairs, 3);
            }
        }
        if (leader) bulk_wait_all();
    }
    fence_before_sync();
    __syncthreads();
    // neither CTA retires while the pair's MMAs, copies or arrivals may still reach its memory
    cluster_sync();
    fence_after_sync();
    if (warp == 1) tmem_dealloc_pair(tbase, TM_COLS);
}

// dW = the sum of the split partials, in slice order
__global__ void __launch_bounds__(256) k_sum_slices(const float *part, float *out, size_t n, int nsplit) {
    for (size_t i = (size_t)blockIdx.x * 256 + threadIdx.x; i < n / 4; i += (size_t)gridDim.x * 256) {
        float4 acc = reinterpret_cast<const float4 *>(part)[i];
        for (int s = 1; s < nsplit; ++s) {
            const float4 x = reinterpret_cast<const float4 *>(part + (size_t)s * n)[i];
            acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
        }
        reinterpret_cast<float4 *>(out)[i] = acc;
    }
}

// ---------------------------------------------------------------- fp32 I/O (CUDA cores)
// D [M][N] = op(A) op(B) (+ C): 64 x 64 tiles, 256 threads, 4 x 4 outputs per thread, K in
// steps of 16 through shared memory.  a_t: A stored [K][M]; b_t: B stored [N][K].
__global__ void __launch_bounds__(256) k_gemm_f32(const float *A, const float *B, const float *Cres, float *D, int M,
                                                  int N, int K, int a_t, int b_t) {
    __shared__ float As[16][64 + 4], Bs[16][64 + 4];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += 16) {
        for (int x = threadIdx.x; x < 16 * 64; x += 256) {
            const int kk = x >> 6, i = x & 63;  // As[kk][i] = op(A)[m0 + i][k0 + kk]
            const int m = m0 + i, k = k0 + kk;
            As[kk][i] = (m < M && k < K) ? (a_t ? A[(size_t)k * M + m] : A[(size_t)m * K + k]) : 0.f;
            const int n = n0 + i;  // Bs[kk][i] = op(B)[k0 + kk][n0 + i]
            Bs[kk][i] = (n < N && k < K) ? (b_t ? B[(size_t)n * K + k] : B[(size_t)k * N + n]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            float av[4], bv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                av[u] = As[kk][ty * 4 + u];
                bv[u] = Bs[kk][tx * 4 + u];
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int w = 0; w < 4; ++w) acc[u][w] += av[u] * bv[w];
        }
        __syncthreads();
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int m = m0 + ty * 4 + u;
        if (m >= M) continue;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const int n = n0 + tx * 4 + w;
            if (n < N) D[(size_t)m * N + n] = acc[u][w] + (Cres ? Cres[(size_t)m * N + n] : 0.f);
        }
    }
}

// ---------------------------------------------------------------- host side
int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
    return n;
}

// One bf16 product.  A: [M][K] (a_mn = 0) or [K][M] (a_mn = 1); B: [N][K] (b_mn = 0) or [K][N]
// (b_mn = 1); D: bf16 [M][N] (+ the residual C), or fp32 d32 with nsplit slices.
int gemm_bf16(const void *A, int a_mn, const void *B, int b_mn, const void *C, void *D, float *d32, int M, int N,
              int K, int nsplit, size_t slice_elems, cudaStream_t s) {
    Maps mp;
    // boxes: one CTA's half of a tile (128 rows of A, D and the residual; 128 columns of B)
    bool ok = a_mn ? make_map_2d_bf16(&mp.a, A, M, K, 64) : make_map_2d_bf16(&mp.a, A, K, M, HM);
    ok = ok && (b_mn ? make_map_2d_bf16(&mp.b, B, N, K, 64) : make_map_2d_bf16(&mp.b, B, K, N, HN));
    mp.c = mp.d = mp.a;  // unused ones keep a valid map
    if (ok && C) ok = make_map_2d_bf16(&mp.c, C, N, M, HM);
    if (ok && D) ok = make_map_2d_bf16(&mp.d, D, N, M, HM);
    if (!ok) return DR_ERR_CUDA;
    Args a;
    a.M = M; a.N = N; a.K = K; a.a_mn = a_mn; a.b_mn = b_mn; a.has_c = C != nullptr;
    a.d32 = d32; a.slice_elems = slice_elems; a.nsplit = nsplit;
    a.kslice = ((K + nsplit - 1) / nsplit + BK - 1) / BK * BK;
    const int tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN) * nsplit;
    int pairs = sm_count() / 2;
    if (pairs <= 0) return DR_ERR_CUDA;
    const size_t smem = SMEM_BYTES + 1024;
    if (cudaFuncSetAttribute(k_gemm_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return DR_ERR_CUDA;
    // persistent: one 2-CTA cluster per pair of SMs, at most one per tile
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(2 * pairs);
    int fit = 0;  // clusters that can be resident at once (a persistent grid must not need a second wave)
    if (cudaOccupancyMaxActiveClusters(&fit, k_gemm_tc, &cfg) == cudaSuccess && fit > 0 && fit < pairs) pairs = fit;
    cfg.gridDim = dim3(2 * (tiles < pairs ? tiles : pairs));
    return cudaLaunchKernelEx(&cfg, k_gemm_tc, mp, a) == cudaSuccess ? DR_OK : DR_ERR_CUDA;
}

int gemm_f32(const float *A, int a_t, const float *B, int b_t, const float *C, float *D, int M, int N, int K,
             cudaStream_t s) {
    const dim3 grid((N + 63) / 64, (M + 63) / 64);
    if (grid.y > 65535) return DR_ERR_UNSUPPORTED;
    k_gemm_f32<<<grid, 256, 0, s>>>(A, B, C, D, M, N, K, a_t, b_t);
    return cudaGetLastError() == cudaSuccess ? DR_OK : DR_ERR_CUDA;
}

}  // namespace clv

size_t clvr_ws_bytes() { return clv::WS; }

int clvr_fwd_run(const void *U, const void *W, const void *h, void *h_out, int M, int K, int N, bool bf16,
                 void *ws, size_t ws_bytes, cudaStream_t s) {
    (void)ws; (void)ws_bytes;
    if (!bf16)
        return clv::gemm_f32((const float *)U, 0, (const float *)W, 0, (const float *)h, (float *)h_out, M, N, K, s);
    // A = U [M][K] (K-major), B = W [K][N] (MN-major)
    return clv::gemm_bf16(U, 0, W, 1, h, h_out, nullptr, M, N, K, 1, 0, s);
}

int clvr_bwd_run(const void *U, const void *W, const void *dH, void *dU, float *dW, int M, int K, int N, bool bf16,
                 void *ws, size_t ws_bytes, cudaStream_t s) {
    if (!bf16) {
        int rc = DR_OK;
        if (dU) rc = clv::gemm_f32((const float *)dH, 0, (const float *)W, 1, nullptr, (float *)dU, M, K, N, s);
        if (rc == DR_OK && dW) rc = clv::gemm_f32((const float *)U, 1, (const float *)dH, 0, nullptr, dW, K, N, M, s);
        return rc;
    }
    if (dU) {  // dU [M][K] = dH [M][N] W^T: A = dH (K-major), B = W [K][N] read as [N'=K][K'=N] (K-major)
        const int rc = clv::gemm_bf16(dH, 0, W, 0, nullptr, dU, nullptr, M, K, N, 1, 0, s);
        if (rc != DR_OK) return rc;
    }
    if (dW) {  // dW [K][N] = U^T dH: A = U [M][K] (MN-major), B = dH [M][N] (MN-major); the M-long
               // reduction in slices with fp32 partials: the slice count that minimises the rounds of
               // work items over the SM pairs times the slice length (fewest slices on a tie), within
               // the workspace
        const size_t elems = (size_t)K * N;
        const int tiles = ((K + clv::BM - 1) / clv::BM) * ((N + clv::BN - 1) / clv::BN), pairs = clv::sm_count() / 2;
        const int kb = (M + clv::BK - 1) / clv::BK;
        int nsplit = 1;
        if (pairs > 0) {
            double best = 0.0;
            for (int ns = 1; ns <= clv::MAX_SPLIT && ns <= (kb > 0 ? kb : 1); ++ns) {
                if (ns > 1 && (size_t)ns * elems * sizeof(float) > ws_bytes) break;
                const double cost = (double)((tiles * ns + pairs - 1) / pairs) * ((kb + ns - 1) / ns);
                if (ns == 1 || cost < best) { best = cost; nsplit = ns; }
            }
        }
        if (nsplit == 1) return clv::gemm_bf16(U, 1, dH, 1, nullptr, nullptr, dW, K, N, M, 1, elems, s);
        float *part = (float *)ws;
        int rc = clv::gemm_bf16(U, 1, dH, 1, nullptr, nullptr, part, K, N, M, nsplit, elems, s);
        if (rc != DR_OK) return rc;
        clv::k_sum_slices<<<148 * 4, 256, 0, s>>>(part, dW, elems, nsplit);
        return cudaGetLastError() == cudaSuccess ? DR_OK : DR_ERR_CUDA;
    }
    return DR_OK;
}

}  // namespace dr
