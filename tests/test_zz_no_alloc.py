"""The forward entry point that allocates nothing: delta_rule_fwd_noalloc.

Callers inside a CUDA graph being captured, allocator-less embedded runtimes and
plugins that receive only their input and output buffers cannot call cudaMalloc,
so they cannot provide the workspace delta_rule_fwd asks for.  This entry point
takes its scratch from a buffer built into the library instead.  Its results
must match delta_rule_fwd's on the same inputs, on consecutive calls that share
that buffer (the second call must not see anything left over by the first).

This file is collected last on purpose; it also passes when run on its own.
"""
import pytest
import torch

from gated_delta_rule_107_b200 import binding
from parity_util import TOL, compare_fwd, gen, np64, oracle_fwd, rel_err

pytestmark = pytest.mark.gpu


def _noalloc(x, variant, dtype_code):
    B, T, H, dk = x["q"].shape
    dv = x["v"].shape[-1]
    out = torch.full_like(x["v"], float("nan"))
    u = torch.full_like(x["v"], float("nan"))
    S_T = torch.full((B, H, dk, dv), float("nan"), device="cuda")
    p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    rc = binding.fwd_noalloc_raw(p(x["q"]), p(x["k"]), p(x["v"]), p(x["loga"]), p(x["beta"]), p(x["S0"]), p(out),
                                 p(u), p(S_T), B, T, H, dk, dv, binding.VARIANTS[variant], 64, dtype_code,
                                 torch.cuda.current_stream().cuda_stream)
    assert rc == binding.DR_OK, binding.strerror(rc)
    torch.cuda.synchronize()
    assert binding.sync_status() == binding.DR_OK
    return {"o": out, "u": u, "S_T": S_T}


@pytest.mark.parametrize("dtype", ("f32", "bf16"))
def test_noalloc_forward_matches_regular_entry_on_two_calls(dtype):
    """At dk = 64 delta_rule_fwd runs the same CUDA-core kernels, so the results are bit-equal;
    both also meet the stated bar against the oracle."""
    code = binding.DR_F32 if dtype == "f32" else binding.DR_BF16
    # two different problems back to back through the same built-in scratch
    for variant, seed, T in (("gdn", 21, 200), ("kda", 22, 130)):
        x = gen(variant, dtype, 2, T, 2, 64, 64, seed=seed, s0_std=0.1)
        o, u, S = binding.delta_rule_fwd(x["q"], x["k"], x["v"], x["loga"], x["beta"], x["S0"], variant=variant)
        torch.cuda.synchronize()
        ref = {"o": o, "u": u, "S_T": S}
        got = _noalloc(x, variant, code)
        for key in ("o", "u", "S_T"):
            assert torch.equal(got[key], ref[key]), f"{variant} {dtype} {key} differs from delta_rule_fwd"
        compare_fwd(got, oracle_fwd(x, variant), dtype, what=f"noalloc {variant} {dtype}")


def test_noalloc_forward_against_tensor_core_forward():
    """At dk = 128 in bf16 delta_rule_fwd takes the tensor-core path; the CUDA-core result of the
    allocation-free entry agrees with it within the bf16 bar, and with the oracle."""
    x = gen("gdn", "bf16", 1, 300, 2, 128, 128, seed=23, s0_std=0.1)
    o, u, S = binding.delta_rule_fwd(x["q"], x["k"], x["v"], x["loga"], x["beta"], x["S0"], variant="gdn")
    torch.cuda.synchronize()
    got = _noalloc(x, "gdn", binding.DR_BF16)
    for key, ref in (("o", o), ("u", u), ("S_T", S)):
        err = rel_err(np64(got[key]), np64(ref))
        assert err <= TOL["bf16"], f"{key}: {err}"
    compare_fwd(got, oracle_fwd(x, "gdn"), "bf16", what="noalloc gdn bf16 d128")


def test_noalloc_rejects_problems_larger_than_its_scratch():
    # 8 x 4096 x 8 at d = 128 needs far more than the built-in 32 MiB
    args = [None] * 9 + [8, 4096, 8, 128, 128, binding.DR_GATED, 64, binding.DR_BF16, None]
    q = torch.empty(16, device="cuda")
    args[0] = args[1] = args[2] = args[3] = args[4] = args[6] = q.data_ptr()
    assert binding.fwd_noalloc_raw(*args) == binding.DR_ERR_WORKSPACE
