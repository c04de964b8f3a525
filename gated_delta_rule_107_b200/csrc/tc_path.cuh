// tc_path.cuh -- the tcgen05 tensor-core path (bf16 I/O, dk = dv = 128, chunk 64).
#pragma once
#include "dr_common.cuh"

namespace dr {

bool tc_fwd_supported(const Geo &g, bool bf16);
size_t tc_fwd_ws_bytes(const Geo &g);
cudaError_t tc_fwd(const Geo &g, const Tensors &t, void *workspace, cudaStream_t s, Rec &rec);
// warp-specialised forward for Gated DeltaNet / DeltaNet (tc_fwd2.cu)
cudaError_t tc_fwd2(const Geo &g, const Tensors &t, cudaStream_t s, Rec &rec);
// Backward recompute on tensor cores (Gated DeltaNet / DeltaNet, same shapes as tc_fwd):
// fills W, U~, g, P, S_n and U of the CUDA-core backward workspace.
struct SimtWs;
bool tc_bwd_recompute_supported(const Geo &g, bool bf16);
cudaError_t tc_bwd_recompute(const Geo &g, const Tensors &t, const SimtWs &w, cudaStream_t s, Rec &rec);
// All intra-chunk gradients on tensor cores (tc_bwd.cu): dq, dk, dv, dbeta, d log alpha.
cudaError_t tc_bwd_chunk(const Geo &g, const Tensors &t, const SimtWs &w, cudaStream_t s, Rec &rec);
// Reverse state chain on tensor cores: dS_{n+1} of every chunk into w.dSn, and dS0.
cudaError_t tc_bwd_reverse(const Geo &g, const Tensors &t, const SimtWs &w, cudaStream_t s, Rec &rec);
// number of launches of tc_fwd and their names
int tc_fwd_launches(const Geo &g, const char **names, int max_names);

}  // namespace dr
