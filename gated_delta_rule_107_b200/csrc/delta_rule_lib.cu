// delta_rule_lib.cu -- single translation unit of libdeltarule.so (the device error
// word and all kernels live in one module, so no relocatable device code is needed).
#include "simt_path.cu"
#include "tc_fwd.cu"
#include "tc_prep.cu"
#include "tc_chain.cu"
#include "tc_bwd.cu"
#include "tc_state.cu"
#include "decode.cu"
#include "prepost.cu"
#include "shortconv.cu"
#include "clvr.cu"
#include "api.cu"
#include "noalloc.cu"
