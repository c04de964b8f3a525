// noalloc.cu -- forward entry point for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at all: code running inside a CUDA graph
// that is being captured, allocator-less embedded runtimes, or plugins that are
// handed only their input and output buffers by a host framework.  For them,
// delta_rule_fwd_noalloc runs the CUDA-core forward (k_prep, k_scan, k_out) with
// its scratch taken from a fixed buffer compiled into this library instead of a
// caller-provided workspace.  Every GPU that loads the library holds the buffer
// until the process exits.
#include <mutex>

#include "../../include/delta_rule.h"
#include "dr_common.cuh"
#include "simt_path.cuh"

namespace dr {

static_assert(DELTA_RULE_NOALLOC_SCRATCH_BYTES % 256 == 0, "scratch size must keep 256-byte alignment");

// The built-in scratch.  In host code this name is only a host-side stand-in:
// its device address must be looked up with cudaGetSymbolAddress on each device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[DELTA_RULE_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_addr[kMaxDevices] = {};

// Device address of the scratch on the current device; looked up once per device.
int noalloc_scratch(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DR_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_addr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return DR_ERR_CUDA;
        }
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return DR_OK;
}

}  // namespace
}  // namespace dr

extern "C" int delta_rule_fwd_noalloc(const void *q, const void *k, const void *v, const void *alpha,
                                      const void *beta, const float *S0, void *out, void *u, float *S_T, int B,
                                      int T, int H, int dk, int dv, int variant, int chunk, int dtype, void *stream) {
    using namespace dr;
    Geo g;
    int rc = check_shape(B, T, H, dk, dv, variant, chunk, dtype, &g);
    if (rc != DR_OK) return rc;
    cudaStream_t s = (cudaStream_t)stream;
    const bool empty = (size_t)B * H == 0;
    if (T == 0 || empty) return empty ? DR_OK : copy_state(S_T, S0, g, s);
    if (!q || !k || !v || !beta || !out) return DR_ERR_ARG;
    if (variant != DR_DELTANET && !alpha) return DR_ERR_ARG;
    const void *ptrs[] = {q, k, v, variant == DR_KDA ? alpha : nullptr, S0, out, u, S_T};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return DR_ERR_ALIGN;
    if (!aligned_elem(beta, dtype) || (variant == DR_GATED && !aligned_elem(alpha, dtype))) return DR_ERR_ALIGN;
    // the CUDA-core forward's scratch must fit the built-in buffer
    if (simt_ws_bytes(g, false) > (size_t)DELTA_RULE_NOALLOC_SCRATCH_BYTES) return DR_ERR_WORKSPACE;
    void *scratch = nullptr;
    rc = noalloc_scratch(&scratch);
    if (rc != DR_OK) return rc;
    Tensors t = {};
    t.q = q; t.k = k; t.v = v; t.alpha = alpha; t.beta = beta; t.S0 = S0; t.out = out; t.u = u; t.S_T = S_T;
    const SimtWs w = simt_ws_carve(g, false, scratch);
    Rec rec;
    return launch_status(simt_fwd(g, t, dtype == DR_BF16, w, s, rec));
}
