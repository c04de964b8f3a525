"""The C-ABI library builds, loads and exports every declared symbol (no GPU needed).

Only argument-validation calls are made here; they return before any CUDA call.
"""
import ctypes
import glob
import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b(delta_rule_\w+)\s*\(", text):
            names.add(m.group(1))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    if shutil.which("nvcc") is None and not os.path.exists(os.path.join(ROOT, "gated_delta_rule_107_b200",
                                                                        "libdeltarule.so")):
        pytest.skip("no nvcc and no prebuilt library")
    from gated_delta_rule_107_b200 import binding, build
    build.build()
    return binding.load()


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert "delta_rule_fwd" in names and "delta_rule_bwd" in names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
    so = os.path.join(ROOT, "gated_delta_rule_107_b200", "libdeltarule.so")
    out = subprocess.run(["nm", "-D", "--defined-only", so], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (delta_rule_\w+)", out))
    assert set(names) <= exported


def test_no_compute_validation_paths(lib):
    from gated_delta_rule_107_b200 import binding
    assert binding.workspace_size(8, 4096, 8, 128, 128, 1, 64, 1, 0) >= 0
    assert binding.workspace_size(8, 4096, 8, 128, 128, 1, 64, 1, 1) > 0
    assert lib.delta_rule_workspace_size(1, 10, 1, 96, 128, 1, 64, 1, 0) == ctypes.c_size_t(-1).value
    assert lib.delta_rule_workspace_size(1, 10, 1, 128, 128, 9, 64, 1, 0) == ctypes.c_size_t(-1).value
    assert lib.delta_rule_workspace_size(1, 10, 1, 128, 128, 1, 0, 1, 0) == ctypes.c_size_t(-1).value
    # invalid enums / shapes are rejected before any CUDA call
    args = [None] * 9 + [1, 10, 1, 128, 128, 7, 64, 1, None, 0, None]
    assert binding.fwd_raw(*args) == binding.DR_ERR_ARG
    args = [None] * 15 + [1, 10, 1, 128, 96, 1, 64, 1, None, 0, None]
    assert binding.bwd_raw(*args) == binding.DR_ERR_UNSUPPORTED
    assert binding.strerror(binding.DR_ERR_TIMEOUT) == "device wait timed out"
    # the saved-activation pair: sizes of the saved buffer and of each call's workspace
    sv = binding.saved_size(8, 4096, 8, 128, 128, 1, 64, 1)
    assert sv > 0 and sv % 256 == 0
    assert binding.workspace_size(8, 4096, 8, 128, 128, 1, 64, 1, 2) == 0
    assert 0 < binding.workspace_size(8, 4096, 8, 128, 128, 1, 64, 1, 3) < binding.workspace_size(
        8, 4096, 8, 128, 128, 1, 64, 1, 1)
    # KDA: the saved buffer holds per chunk g|beta (512 B), W, U~, U, q e^g, k e^{g_C - g} (16 KiB
    # each), P, T and the gated k k^T (8 KiB each), e^{g_C} (512 B), the chunk flag (4 B), the state
    # entering the chunk and the fp32 gate (32 KiB each)
    n_chunks = 8 * 16 * 64
    assert binding.saved_size(8, 4096, 16, 128, 128, 2, 64, 1) == n_chunks * (
        512 + 5 * 16384 + 3 * 8192 + 512 + 4 + 2 * 32768)
    assert 0 < binding.workspace_size(8, 4096, 16, 128, 128, 2, 64, 1, 3) < binding.workspace_size(
        8, 4096, 16, 128, 128, 2, 64, 1, 1)
    assert binding.saved_size(1, 256, 2, 64, 64, 0, 64, 0) == 0       # fp32 I/O: no saved form
    assert binding.saved_size(1, 256, 2, 64, 64, 2, 64, 1) == 0       # d = 64: no saved form
    assert lib.delta_rule_workspace_size(1, 10, 1, 128, 128, 1, 64, 1, 4) == ctypes.c_size_t(-1).value
    assert lib.delta_rule_saved_size(1, 10, 1, 96, 128, 1, 64, 1) == ctypes.c_size_t(-1).value
    args = [None] * 9 + [1, 10, 1, 128, 128, 7, 64, 1, None, 0, None, 0, None]
    assert binding.fwd_save_raw(*args) == binding.DR_ERR_ARG
    assert binding.strerror(12345) == "unknown error code"


def test_operations_around_the_core_validate_before_any_launch(lib):
    """The short convolution, the routing products, decoding and the pre/post operations reject bad
    shapes, enums and pointers with their codes, and size their workspaces, without a GPU."""
    from gated_delta_rule_107_b200 import binding
    bad = ctypes.c_size_t(-1).value
    # short convolution: D a multiple of 8; workspace = one fp32 [D][4] partial per (sequence, 64 tokens)
    assert lib.delta_rule_shortconv_workspace_size(8, 4096, 1024) == 8 * 64 * 1024 * 4 * 4
    assert lib.delta_rule_shortconv_workspace_size(2, 0, 64) == 2 * 1 * 64 * 4 * 4
    assert lib.delta_rule_shortconv_workspace_size(1, 10, 60) == bad
    assert binding.shortconv_raw(None, None, None, None, None, 1, 10, 60, binding.DR_BF16, None) == \
        binding.DR_ERR_UNSUPPORTED
    assert binding.shortconv_raw(None, None, None, None, None, 1, 10, 64, 3, None) == binding.DR_ERR_ARG
    assert binding.shortconv_raw(None, None, None, None, None, -1, 10, 64, binding.DR_BF16, None) == binding.DR_ERR_ARG
    assert binding.shortconv_raw(None, None, None, None, None, 0, 10, 64, binding.DR_BF16, None) == binding.DR_OK
    assert binding.shortconv_raw(None, None, None, None, None, 1, 10, 64, binding.DR_BF16, None) == binding.DR_ERR_ARG
    assert binding.shortconv_bwd_raw(None, None, None, None, None, None, None, 1, 10, 64, binding.DR_BF16, None, 0,
                                     None) == binding.DR_ERR_ARG
    # routing: K, N multiples of 8, a caller workspace, M = 0 a no-op
    assert lib.delta_rule_clvr_workspace_size() >= 1 << 20
    assert binding.clvr_raw(None, None, None, None, 4, 60, 64, binding.DR_BF16, None, 0, None) == \
        binding.DR_ERR_UNSUPPORTED
    assert binding.clvr_raw(None, None, None, None, 4, 64, 64, 7, None, 0, None) == binding.DR_ERR_ARG
    assert binding.clvr_raw(None, None, None, None, 0, 64, 64, binding.DR_BF16, None, 0, None) == binding.DR_OK
    assert binding.clvr_raw(None, None, None, None, 4, 64, 64, binding.DR_BF16, None, 0, None) == binding.DR_ERR_ARG
    assert binding.clvr_bwd_raw(None, None, None, None, None, 4, 64, 64, binding.DR_BF16, None, 0, None) == \
        binding.DR_ERR_ARG
    # decoding and the pre/post operations
    assert binding.decode_raw(*([None] * 9), 1, 2, 1, 96, 128, binding.DR_GATED, binding.DR_BF16, None) == \
        binding.DR_ERR_UNSUPPORTED
    assert binding.preop_raw(*([None] * 8), 1, 4, 1, 96, binding.DR_GATED, binding.DR_BF16, None) == \
        binding.DR_ERR_UNSUPPORTED
    assert binding.postop_raw(None, None, None, None, 1, 4, 1, 128, 5, None) == binding.DR_ERR_ARG
    assert lib.delta_rule_postop_workspace_size(96) == bad


def test_launch_plans(lib):
    """Which kernels each call launches (host logic, no GPU): the tensor-core paths for bf16 at
    d = 128, the KDA hybrid backward, the fused dv = 64 kernel and the CUDA-core path."""
    from gated_delta_rule_107_b200 import binding
    split = {0: ["k_chunk_prep", "k_chain_fwd"],
             1: ["k_chunk_prep(keep)", "k_chain_fwd(recompute)", "k_chain_rev", "k_bwd_chunk_tc"],
             2: ["k_chunk_prep(keep)", "k_chain_fwd(keep)"],
             3: ["k_chain_rev", "k_bwd_chunk_tc"]}
    for variant in (0, 1):
        for kind, names in split.items():
            assert binding.launches(8, 4096, 8, 128, 128, variant, 64, 1, kind) == names
    kda_split = ["k_kda_gates", "k_kda_diag", "k_chunk_prep", "k_chain_fwd"]
    assert binding.launches(4, 16384, 8, 128, 128, 2, 64, 1, 0) == kda_split
    assert binding.launches(4, 16384, 8, 128, 128, 2, 64, 1, 2) == kda_split[:2] + ["k_chunk_prep(keep)",
                                                                                   "k_chain_fwd(keep)"]
    # the tensor-core intra-chunk gradient, then the CUDA-core one for chunks past the block split's range
    kda_bwd = ["k_kda_gates", "k_kda_diag", "k_chunk_prep(keep)", "k_chain_fwd(recompute)", "k_chain_rev",
               "k_bwd_kda_tc", "k_widen", "k_widen", "k_state_tc", "k_bwd_intra"]
    assert binding.launches(8, 4096, 16, 128, 128, 2, 64, 1, 1) == kda_bwd
    assert binding.launches(8, 4096, 16, 128, 128, 2, 64, 1, 3) == kda_bwd[4:]  # from saved: no recompute
    # KDA at dv = 64 takes the CUDA-core forward; the fused dv = 64 kernel serves scalar gates
    assert binding.launches(2, 512, 4, 128, 64, 2, 64, 1, 0) == ["k_prep", "k_scan", "k_out"]
    assert binding.launches(2, 512, 4, 128, 64, 1, 64, 1, 0) == ["k_fwd_tc"]
    assert binding.launches(1, 256, 2, 64, 64, 0, 64, 0, 0) == ["k_prep", "k_scan", "k_out"]
    assert binding.launches(1, 256, 2, 64, 64, 0, 64, 0, 1) == ["k_prep", "k_scan", "k_scan_bwd", "k_bwd_state",
                                                             "k_bwd_intra"]
