// tc_tile.cuh -- small helpers for 128B-swizzled bf16 tiles and TMEM rows.
#pragma once
#include "tc_ptx.cuh"

namespace dr {
namespace tcf {

using namespace dr::tc;

__device__ __forceinline__ float bf(const void *p, size_t i) {
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i]);
}

__device__ __forceinline__ void st_chunk(unsigned char *base, uint32_t off, const float *v) {
    uint4 w;
    w.x = pack_bf16(v[0], v[1]);
    w.y = pack_bf16(v[2], v[3]);
    w.z = pack_bf16(v[4], v[5]);
    w.w = pack_bf16(v[6], v[7]);
    *reinterpret_cast<uint4 *>(base + off) = w;
}

__device__ __forceinline__ void ld_chunk(const unsigned char *base, uint32_t off, float *v) {
    const uint4 w = *reinterpret_cast<const uint4 *>(base + off);
    v[0] = bf16_lo(w.x); v[1] = bf16_hi(w.x); v[2] = bf16_lo(w.y); v[3] = bf16_hi(w.y);
    v[4] = bf16_lo(w.z); v[5] = bf16_hi(w.z); v[6] = bf16_lo(w.w); v[7] = bf16_hi(w.w);
}

// 64 fp32 columns of this thread's TMEM lane
__device__ __forceinline__ void tmem_row64(uint32_t taddr, float *v) {
    tmem_ld16(taddr + 0, v);
    tmem_ld16(taddr + 16, v + 16);
    tmem_ld16(taddr + 32, v + 32);
    tmem_ld16(taddr + 48, v + 48);
    wait_ld();
}

}  // namespace tcf
}  // namespace dr
