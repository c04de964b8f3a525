// tc_fwd.cu -- tcgen05 forward (not yet enabled: every call takes the CUDA-core path).
#include "tc_path.cuh"

namespace dr {

bool tc_fwd_supported(const Geo &, bool) { return false; }
size_t tc_fwd_ws_bytes(const Geo &) { return 0; }
cudaError_t tc_fwd(const Geo &, const Tensors &, void *, cudaStream_t, Rec &) { return cudaErrorNotSupported; }
int tc_fwd_launches(const char **, int) { return 0; }

}  // namespace dr
