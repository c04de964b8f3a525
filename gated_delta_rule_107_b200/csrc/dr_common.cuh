// dr_common.cuh -- shared device helpers and argument structs of libdeltarule.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace dr {

enum : int { VAR_DELTANET = 0, VAR_GATED = 1, VAR_KDA = 2 };

// Device error word: set by kernels whose bounded waits expire; read and cleared
// by delta_rule_sync_status().  Bit values below.  The library is one translation
// unit (delta_rule_lib.cu), so this is the only definition.
enum : int { DEVERR_TIMEOUT = 1 };
__device__ int g_dev_error = 0;

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

// Problem geometry shared by all kernels.  N = number of chunks = ceil(T / C).
struct Geo {
    int B, T, H, dk, dv, C, N, variant;
    // element offset of token row (b, t, h) in a [B,T,H,*] tensor, before the *d
    __host__ __device__ __forceinline__ size_t row(int b, int t, int h) const {
        return ((size_t)b * T + t) * H + h;
    }
    // index of chunk n of (b, h) in chunk-major workspaces [B,H,N,...]
    __host__ __device__ __forceinline__ size_t chunk(int b, int h, int n) const {
        return ((size_t)b * H + h) * N + n;
    }
};

// Forward / backward tensor arguments (device pointers; see include/delta_rule.h).
struct Tensors {
    const void *q, *k, *v, *alpha, *beta;
    const float *S0;
    void *out, *u;
    float *S_T;
    const void *dout, *du;
    const float *dS_T;
    void *dq, *dk, *dv, *dalpha, *dbeta;
    float *dS0;
    // the fused forward (delta_rule_fwd_fused): q, k, alpha, beta hold the raw projections and
    // logits; the post-operation's gate logits and weight, and its output y
    const void *gate_o;
    const float *w_norm;
    void *y;
};

// Optional launch timing: records ev[i] on the stream just before kernel launch i
// and ev[n_launches] after the last one (the *_timed entry points).  Inactive
// when ev is null.
struct Rec {
    cudaEvent_t *ev = nullptr;
    int n = 0, i = 0;
    bool bad = false;  // an event could not be recorded (invalid handle)
    void mark(cudaStream_t s) {
        if (ev && i < n && cudaEventRecord(ev[i++], s) != cudaSuccess) {
            cudaGetLastError();  // consume it: it is not a launch failure
            bad = true;
        }
    }
};

}  // namespace dr
