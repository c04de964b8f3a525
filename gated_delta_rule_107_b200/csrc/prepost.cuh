// prepost.cuh -- the pre- and post-operations around the core (prepost.cu).
#pragma once
#include "dr_common.cuh"

namespace dr {

// Arguments of one pre/post call (device pointers; rows = B * T * H, d = dk or dv).
//   pre  forward:  q, k, b, a -> qo, ko, bo, ao
//   pre  backward: q, k, b, a and dq, dk, db, da (gradients of qo, ko, bo, ao) -> qo, ko, bo, ao
//   post forward:  q = o, k = g, w -> qo = y
//   post backward: q = o, k = g, w, dq = dy -> qo = do, ko = dg, dw (part = workspace)
struct PrePost {
    const void *q, *k, *b, *a;
    const void *dq, *dk, *db, *da;
    void *qo, *ko, *bo, *ao;
    const float *w;
    float *dw, *part;
    size_t rows;
    int d, variant;
};
size_t postop_ws_bytes(int dv);
cudaError_t preop_run(const PrePost &p, bool bf16, bool bwd, cudaStream_t s);
cudaError_t postop_run(const PrePost &p, bool bf16, bool bwd, cudaStream_t s);

}  // namespace dr
