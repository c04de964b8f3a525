// shortconv.cuh -- the depthwise causal short convolution before the core (shortconv.cu).
#pragma once
#include "dr_common.cuh"

namespace dr {

// One short-convolution call (device pointers): x, y, dy, dx [B, T, D]; cin, cout, dcin [B, 3, D];
// w, dw [D][4] fp32; part = workspace of the backward's dw partials.
struct ShortConv {
    const void *x, *cin, *dy;
    void *y, *cout, *dx, *dcin;
    const float *w;
    float *dw, *part;
    int B, T, D;
};
size_t shortconv_ws_bytes(int B, int T, int D);
// grid size (CTAs) of the forward or backward pass; 0 when the shape needs none
long long shortconv_ctas(int B, int T, int D, bool bf16, bool bwd);
cudaError_t shortconv_run(const ShortConv &p, bool bf16, bool bwd, cudaStream_t s);

}  // namespace dr
