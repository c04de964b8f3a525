// tc_probe.cu -- GPU self-checks of the tcgen05 / TMA building blocks in
// gated_delta_rule_107_b200/csrc/tc_ptx.cuh (test infrastructure).
//
// probe_mma: D = (-1)^neg_a A (M x K) . B (K x N) (+ the same again when
// accumulate) with A and B staged in the swizzled canonical layouts (K-major or
// MN-major) exactly as the fused kernel stages them; D read back with
// tcgen05.ld.  probe_tma: one 4-D TMA box load, read back through the swizzle
// helper.  Operands sit at the start of a 227 KB shared allocation so that any
// misread of the layout stays inside it.
#include <stdio.h>

#include "../../gated_delta_rule_107_b200/csrc/dr_common.cuh"
#include "../../gated_delta_rule_107_b200/csrc/tc_host.cuh"
#include "../../gated_delta_rule_107_b200/csrc/tc_inverse.cuh"
#include "../../gated_delta_rule_107_b200/csrc/tc_ptx.cuh"

using namespace dr;
using namespace dr::tc;

static constexpr int SMEM = 200 * 1024;  // + 1 KB static stays under the 227 KB limit
static constexpr int B_OFF = 96 * 1024;

// element (row, col) of a panelled swizzled tile whose rows are `rows` long in
// units of 64-element panels; panel p of width 64 starts at p * panel_bytes.
__device__ __forceinline__ uint32_t tile_off(int row, int col, uint32_t panel_bytes) {
    return (col >> 6) * panel_bytes + swz(row, (col & 63) >> 3) + (col & 7) * 2;
}

__global__ void k_probe_mma(const __nv_bfloat16 *A, const __nv_bfloat16 *B, float *D, int M, int N, int K, int a_mn,
                            int b_mn, int neg_a, int accumulate, int *status) {
    extern __shared__ __align__(1024) unsigned char sm[];
    __shared__ uint64_t bar;
    __shared__ uint32_t tbase;
    __shared__ int abort_flag;
    const int tid = threadIdx.x, warp = tid >> 5;
    unsigned char *sa = sm, *sb = sm + B_OFF;
    // stage A: K-major -> rows m, K along panels (panel = M rows x 128 B);
    //          MN-major -> rows k, M along panels (panel = K rows x 128 B)
    for (int x = tid; x < M * K; x += blockDim.x) {
        const int m = x / K, k = x % K;
        const uint32_t off = a_mn ? tile_off(k, m, (uint32_t)K * 128) : tile_off(m, k, (uint32_t)M * 128);
        *reinterpret_cast<__nv_bfloat16 *>(sa + off) = A[x];
    }
    for (int x = tid; x < K * N; x += blockDim.x) {
        const int k = x / N, n = x % N;
        const uint32_t off = b_mn ? tile_off(k, n, (uint32_t)K * 128) : tile_off(n, k, (uint32_t)N * 128);
        *reinterpret_cast<__nv_bfloat16 *>(sb + off) = B[x];
    }
    if (tid == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    fence_proxy_async();
    __syncthreads();
    if (warp == 0) tmem_alloc(&tbase, 256);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tm = tbase;
    if (tid == 0) {
        const uint32_t idesc = idesc_bf16(M, N, a_mn, b_mn, neg_a, 0);
        const uint32_t a0 = smem_u32(sa), b0 = smem_u32(sb);
        for (int rep = 0; rep < (accumulate ? 2 : 1); ++rep) {
            for (int s = 0; s < K / 16; ++s) {
                uint64_t ad, bd;
                if (a_mn) ad = sdesc(a0 + s * 2048, (M > 64) ? K * 128 : 1024, 1024);
                else ad = sdesc(a0 + (s >> 2) * M * 128 + (s & 3) * 32, 16, 1024);
                if (b_mn) bd = sdesc(b0 + s * 2048, (N > 64) ? K * 128 : 1024, 1024);
                else bd = sdesc(b0 + (s >> 2) * N * 128 + (s & 3) * 32, 16, 1024);
                mma_bf16(tm, ad, bd, idesc, (rep > 0 || s > 0) ? 1 : 0);
            }
        }
        mma_commit(&bar);
    }
    const bool ok = mbar_wait(&bar, 0, &abort_flag);
    fence_after_sync();
    if (ok) {
        const int lane_base = (warp & 3) * 32;
        const int row = lane_base + (tid & 31);
        for (int c = 0; c < N; c += 16) {
            float v[16];
            tmem_ld16(tm + ((uint32_t)lane_base << 16) + c, v);
            wait_ld();
            if (row < M)
                for (int i = 0; i < 16; ++i) D[row * N + c + i] = v[i];
        }
    } else if (tid == 0) {
        *status = 1;
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tm, 256);
}

__global__ void k_probe_tma(const __grid_constant__ CUtensorMap map, __nv_bfloat16 *out, int c0, int h, int t0, int b,
                            int *status) {
    extern __shared__ __align__(1024) unsigned char sm[];
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    const int tid = threadIdx.x;
    if (tid == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        mbar_arrive_tx(&bar, 64 * 64 * 2);
        tma_load_4d(sm, &map, c0, h, t0, b, &bar);
    }
    if (!mbar_wait(&bar, 0, &abort_flag)) {
        if (tid == 0) *status = 1;
        return;
    }
    for (int x = tid; x < 64 * 64; x += blockDim.x) {
        const int r = x / 64, c = x % 64;
        out[x] = *reinterpret_cast<const __nv_bfloat16 *>(sm + swz(r, c >> 3) + (c & 7) * 2);
    }
}

extern "C" int probe_mma(const void *A, const void *B, float *D, int M, int N, int K, int a_mn, int b_mn, int neg_a,
                         int accumulate) {
    int *st;
    cudaMalloc(&st, sizeof(int));
    cudaMemset(st, 0, sizeof(int));
    cudaFuncSetAttribute(k_probe_mma, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    k_probe_mma<<<1, 128, SMEM>>>((const __nv_bfloat16 *)A, (const __nv_bfloat16 *)B, D, M, N, K, a_mn, b_mn, neg_a,
                                  accumulate, st);
    cudaError_t e = cudaDeviceSynchronize();
    int h = -1;
    cudaMemcpy(&h, st, sizeof(int), cudaMemcpyDeviceToHost);
    cudaFree(st);
    if (e != cudaSuccess) {
        fprintf(stderr, "probe_mma: %s\n", cudaGetErrorString(e));
        return -100;
    }
    return h;
}

extern "C" int probe_tma(const void *X, void *out, int Bn, int T, int H, int d, int b, int h, int t0, int c0) {
    CUtensorMap map;
    if (!make_map_4d_bf16(&map, X, (uint64_t)d, (uint64_t)H, (uint64_t)T, (uint64_t)Bn, 64)) return -200;
    int *st;
    cudaMalloc(&st, sizeof(int));
    cudaMemset(st, 0, sizeof(int));
    cudaFuncSetAttribute(k_probe_tma, cudaFuncAttributeMaxDynamicSharedMemorySize, 16 * 1024);
    k_probe_tma<<<1, 128, 16 * 1024>>>(map, (__nv_bfloat16 *)out, c0, h, t0, b, st);
    cudaError_t e = cudaDeviceSynchronize();
    int hs = -1;
    cudaMemcpy(&hs, st, sizeof(int), cudaMemcpyDeviceToHost);
    cudaFree(st);
    if (e != cudaSuccess) {
        fprintf(stderr, "probe_tma: %s\n", cudaGetErrorString(e));
        return -100;
    }
    return hs;
}

// probe_inverse: T = (I + A)^-1 of a strictly lower-triangular 64 x 64 A (row-major fp32)
// by the warpgroup routine of tc_inverse.cuh.
__global__ void k_probe_inverse(const float *A, float *T) {
    __shared__ float sA[4096], sT[4096], ys[768];
    const int tid = threadIdx.x;
    for (int x = tid; x < 4096; x += 128) {
        sA[sw64(x >> 6, x & 63)] = A[x];
        sT[x] = 0.f;
    }
    __syncthreads();
    unit_lower_inverse64(sA, sT, ys, tid, [] { __syncthreads(); });
    for (int x = tid; x < 4096; x += 128) T[x] = sT[sw64(x >> 6, x & 63)];
}

extern "C" int probe_inverse(const float *A, float *T) {
    k_probe_inverse<<<1, 128>>>(A, T);
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        fprintf(stderr, "probe_inverse: %s\n", cudaGetErrorString(e));
        return -100;
    }
    return 0;
}
