// tc_inverse.cuh -- inverse of the 64 x 64 unit lower-triangular matrix I + A of one
// chunk (the UT transform of "线性注意力架构演进与Kimi Delta Attention创新实践", section
// 6.2), by one warpgroup (128 threads), in fp32 shared memory.
//
// Blocks of 16: L = I + A, T = L^-1.
//   diagonal blocks  T_RR = L_RR^-1        right-looking substitution, 16 lanes per block
//   below diagonal   T_RI = -T_RR (sum_{J=I}^{R-1} L_RJ T_JI)
// Column block I only needs blocks of the same column and the diagonal, so the three
// column chains (I = 0, 1, 2) run on three warps without further synchronisation; each
// 16 x 16 x 16 product is four warp-level tf32 MMAs (m16n8k8) with fp32 accumulation.
#pragma once
#include <stdint.h>

namespace dr {
namespace tc {

// fp32 64 x 64 tile with an XOR swizzle of 4-float groups by the row (conflict-free
// float4 row writes by threads that each own one row, and conflict-free A-fragment
// reads of the warp-level MMAs below).
__device__ __forceinline__ int sw64(int r, int c) { return r * 64 + (c ^ ((r & 7) << 2)); }

__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void mma_tf32_16816(float *d, const uint32_t *a, const uint32_t *b) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// z (two n-tiles of the m16n8 fragment) += X[xr.., xc..] (16x16) . Y[yr.., yc..] (16x16)
// X, Y: swizzled fp32 64 x 64 tiles.
__device__ __forceinline__ void mm16_acc(float (*z)[4], const float *X, int xr, int xc, const float *Y, int yr, int yc,
                                         int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
        uint32_t a[4];
        a[0] = to_tf32(X[sw64(xr + g, xc + 8 * kk + t)]);
        a[1] = to_tf32(X[sw64(xr + g + 8, xc + 8 * kk + t)]);
        a[2] = to_tf32(X[sw64(xr + g, xc + 8 * kk + t + 4)]);
        a[3] = to_tf32(X[sw64(xr + g + 8, xc + 8 * kk + t + 4)]);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            uint32_t b[2];
            b[0] = to_tf32(Y[sw64(yr + 8 * kk + t, yc + 8 * nt + g)]);
            b[1] = to_tf32(Y[sw64(yr + 8 * kk + t + 4, yc + 8 * nt + g)]);
            mma_tf32_16816(z[nt], a, b);
        }
    }
}

// Store sign * z (fragment layout) into the 16 x 16 block of swizzled tile Z at (zr, zc).
__device__ __forceinline__ void st16(float *Z, int zr, int zc, float (*z)[4], float sign, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        Z[sw64(zr + g, zc + 8 * nt + 2 * t)] = sign * z[nt][0];
        Z[sw64(zr + g, zc + 8 * nt + 2 * t + 1)] = sign * z[nt][1];
        Z[sw64(zr + g + 8, zc + 8 * nt + 2 * t)] = sign * z[nt][2];
        Z[sw64(zr + g + 8, zc + 8 * nt + 2 * t + 1)] = sign * z[nt][3];
    }
}

// T = (I + A)^-1 for strictly lower-triangular A.  A, T: swizzled fp32 64 x 64 tiles;
// Ysc: 3 x 256 floats of per-warp scratch.  wt: thread index in the warpgroup (0..127);
// sync(): barrier over the warpgroup.  On return T holds the full lower triangle
// (diagonal ones included) and zeros above the diagonal in every diagonal block;
// blocks above the block diagonal are not written.
template <typename Sync>
__device__ __forceinline__ void unit_lower_inverse64(const float *A, float *T, float *Ysc, int wt, Sync sync) {
    const int warp = wt >> 5, lane = wt & 31;
    // diagonal blocks: lane j (< 16) of warp R owns column j of T_RR; the strictly lower part
    // of L_RR is read into registers first (float4 groups stay whole under sw64)
    if (lane < 16) {
        const int R = warp, j = lane, o = 16 * R;
        float a[16][16];
#pragma unroll
        for (int r = 1; r < 16; ++r) {
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                if (4 * c4 < r) {
                    const float4 v = *reinterpret_cast<const float4 *>(&A[sw64(o + r, o + 4 * c4)]);
                    a[r][4 * c4] = v.x; a[r][4 * c4 + 1] = v.y; a[r][4 * c4 + 2] = v.z; a[r][4 * c4 + 3] = v.w;
                }
            }
        }
        float t[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) t[r] = (r == j) ? 1.f : 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
#pragma unroll
            for (int r = i + 1; r < 16; ++r) t[r] -= a[r][i] * t[i];
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) T[sw64(o + r, o + j)] = t[r];
    }
    sync();
    // column chains: warp I computes T_RI for R = I+1 .. 3
    if (warp < 3) {
        const int I = warp;
        float *Y = Ysc + 256 * warp;  // 16 x 16, row-major
        const int g = lane >> 2, t = lane & 3;
        for (int R = I + 1; R < 4; ++R) {
            float z[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            for (int J = I; J < R; ++J) mm16_acc(z, A, 16 * R, 16 * J, T, 16 * J, 16 * I, lane);
            // Y -> scratch (row-major 16 x 16) so it can be read back as the B operand
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                Y[g * 16 + 8 * nt + 2 * t] = z[nt][0];
                Y[g * 16 + 8 * nt + 2 * t + 1] = z[nt][1];
                Y[(g + 8) * 16 + 8 * nt + 2 * t] = z[nt][2];
                Y[(g + 8) * 16 + 8 * nt + 2 * t + 1] = z[nt][3];
            }
            __syncwarp();
            float w[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
                uint32_t a[4];
                const int o = 16 * R;
                a[0] = to_tf32(T[sw64(o + g, o + 8 * kk + t)]);
                a[1] = to_tf32(T[sw64(o + g + 8, o + 8 * kk + t)]);
                a[2] = to_tf32(T[sw64(o + g, o + 8 * kk + t + 4)]);
                a[3] = to_tf32(T[sw64(o + g + 8, o + 8 * kk + t + 4)]);
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    uint32_t b[2];
                    b[0] = to_tf32(Y[(8 * kk + t) * 16 + 8 * nt + g]);
                    b[1] = to_tf32(Y[(8 * kk + t + 4) * 16 + 8 * nt + g]);
                    mma_tf32_16816(w[nt], a, b);
                }
            }
            st16(T, 16 * R, 16 * I, w, -1.f, lane);
            __syncwarp();
        }
    }
    sync();
}

}  // namespace tc
}  // namespace dr
