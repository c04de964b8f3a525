"""B200-native (sm_100a) chunkwise gated delta rule: DeltaNet, Gated DeltaNet, KDA.

The computation lives in ``libdeltarule.so`` (CUDA, C ABI in include/delta_rule.h);
``binding`` marshals torch tensors into that ABI; ``inputs`` draws the seeded
synthetic workloads; ``build`` compiles the library in-tree with nvcc.
"""
from .binding import (DR_BF16, DR_DELTANET, DR_F32, DR_GATED, DR_KDA, DeltaRuleError, delta_rule_bwd,  # noqa: F401
                      delta_rule_fwd, delta_rule_fwd_host)
