"""The training pair: delta_rule_fwd_save keeps what the backward would recompute, and
delta_rule_bwd_saved starts from it.

Both must give exactly the results of the plain forward and the recomputing backward
(the same kernels produce the saved values), and those match the fp64 oracle.
"""
import pytest
import torch

from gated_delta_rule_107_b200 import binding
from parity_util import compare_bwd, gen, gpu_bwd, gpu_fwd, oracle_bwd

pytestmark = pytest.mark.gpu


def _save_pair(x, variant):
    o, u, S, saved = binding.delta_rule_fwd_save(x["q"], x["k"], x["v"], x["loga"], x["beta"], x["S0"],
                                                 variant=variant)
    g = binding.delta_rule_bwd_saved(x["q"], x["k"], x["v"], x["loga"], x["beta"], x["S0"], x["dO"], x.get("du"),
                                     x.get("dS_T"), saved=saved, variant=variant)
    torch.cuda.synchronize()
    assert binding.sync_status() == binding.DR_OK
    return {"o": o, "u": u, "S_T": S}, g, saved


@pytest.mark.parametrize("variant", ("gdn", "deltanet"))
@pytest.mark.parametrize("T,du,s0", ((64, True, 0.0), (130, False, 0.1), (257, True, 0.1)))
def test_saved_pair_equals_recompute_and_oracle(variant, T, du, s0):
    x = gen(variant, "bf16", 2, T, 3, 128, 128, seed=31 + T, s0_std=s0, grads=True, du=du)
    fwd_ref, bwd_ref = gpu_fwd(x, variant), gpu_bwd(x, variant)
    fwd, g, saved = _save_pair(x, variant)
    assert saved is not None and saved.numel() == binding.saved_size(2, T, 3, 128, 128, binding.VARIANTS[variant],
                                                                       64, binding.DR_BF16)
    for key in ("o", "u", "S_T"):
        assert torch.equal(fwd[key], fwd_ref[key]), key
    for key, t in g.items():
        if t is not None:
            assert torch.equal(t, bwd_ref[key]), key
    compare_bwd(g, oracle_bwd(x, variant), "bf16", variant, what=f"saved {variant} T={T}")


def test_configurations_without_a_saved_form_run_the_plain_calls():
    # d = 64 and fp32 I/O have no saved form: saved_size is 0 and the pair equals fwd / bwd
    for variant, dtype, code in (("kda", "bf16", binding.DR_BF16), ("gdn", "f32", binding.DR_F32)):
        x = gen(variant, dtype, 1, 100, 2, 64, 64, seed=41, grads=True)
        assert binding.saved_size(1, 100, 2, 64, 64, binding.VARIANTS[variant], 64, code) == 0
        fwd, g, saved = _save_pair(x, variant)
        assert saved is None
        fwd_ref, bwd_ref = gpu_fwd(x, variant), gpu_bwd(x, variant)
        for key in ("o", "u", "S_T"):
            assert torch.equal(fwd[key], fwd_ref[key]), (variant, key)
        for key, t in g.items():
            if t is not None:
                assert torch.equal(t, bwd_ref[key]), (variant, key)


def test_saved_buffer_is_checked():
    B, T, H, d = 1, 70, 2, 128
    x = gen("gdn", "bf16", B, T, H, d, d, seed=43, grads=True)
    need = binding.saved_size(B, T, H, d, d, binding.DR_GATED, 64, binding.DR_BF16)
    assert need > 0
    buf = torch.empty(need + 512, dtype=torch.uint8, device="cuda")
    o, u, S = (torch.empty_like(x["v"]), torch.empty_like(x["v"]), torch.empty(B, H, d, d, device="cuda"))
    p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    stream = torch.cuda.current_stream().cuda_stream

    def fwd_save(ptr, nbytes):
        return binding.fwd_save_raw(p(x["q"]), p(x["k"]), p(x["v"]), p(x["loga"]), p(x["beta"]), None, p(o), p(u),
                                    p(S), B, T, H, d, d, binding.DR_GATED, 64, binding.DR_BF16, ptr, nbytes, None, 0,
                                    stream)

    assert fwd_save(None, 0) == binding.DR_ERR_WORKSPACE
    assert fwd_save(buf.data_ptr(), need - 1) == binding.DR_ERR_WORKSPACE
    assert fwd_save(buf.data_ptr() + 16, need) == binding.DR_ERR_ALIGN
    assert fwd_save(buf.data_ptr(), need) == binding.DR_OK
    torch.cuda.synchronize()
    g = {k: torch.empty_like(x[s]) for k, s in (("dq", "q"), ("dk", "k"), ("dv", "v"), ("dalpha", "loga"),
                                                 ("dbeta", "beta"))}
    wneed = binding.workspace_size(B, T, H, d, d, binding.DR_GATED, 64, binding.DR_BF16, 3)
    ws = torch.empty(wneed, dtype=torch.uint8, device="cuda")

    def bwd_saved(ptr, nbytes):
        return binding.bwd_saved_raw(p(x["q"]), p(x["k"]), p(x["v"]), p(x["loga"]), p(x["beta"]), None, p(x["dO"]),
                                     None, None, p(g["dq"]), p(g["dk"]), p(g["dv"]), p(g["dalpha"]), p(g["dbeta"]),
                                     None, B, T, H, d, d, binding.DR_GATED, 64, binding.DR_BF16, ptr, nbytes,
                                     ws.data_ptr(), wneed, stream)

    assert bwd_saved(None, 0) == binding.DR_ERR_WORKSPACE
    assert bwd_saved(buf.data_ptr(), need) == binding.DR_OK
    torch.cuda.synchronize()
    assert binding.sync_status() == binding.DR_OK


def test_saved_pair_headline_shape_equals_recompute():
    """B=8, T=4096, H=8, d=128 Gated DeltaNet: the training pair bit-equals fwd + recomputing bwd."""
    x = gen("gdn", "bf16", 8, 4096, 8, 128, 128, seed=1002, grads=True, du=True)
    fwd_ref, bwd_ref = gpu_fwd(x, "gdn"), gpu_bwd(x, "gdn")
    fwd, g, _ = _save_pair(x, "gdn")
    for key in ("o", "u", "S_T"):
        assert torch.equal(fwd[key], fwd_ref[key]), key
    for key, t in g.items():
        if t is not None:
            assert torch.equal(t, bwd_ref[key]), key


@pytest.mark.parametrize("T,du,s0", ((64, True, 0.0), (130, False, 0.1), (257, True, 0.1)))
def test_kda_saved_pair_equals_recompute_and_oracle(T, du, s0):
    x = gen("kda", "bf16", 2, T, 3, 128, 128, seed=61 + T, s0_std=s0, grads=True, du=du)
    fwd_ref, bwd_ref = gpu_fwd(x, "kda"), gpu_bwd(x, "kda")
    fwd, g, saved = _save_pair(x, "kda")
    assert saved is not None and saved.numel() == binding.saved_size(2, T, 3, 128, 128, binding.DR_KDA, 64,
                                                                       binding.DR_BF16)
    for key in ("o", "u", "S_T"):
        assert torch.equal(fwd[key], fwd_ref[key]), key
    for key, t in g.items():
        if t is not None:
            assert torch.equal(t, bwd_ref[key]), key
    compare_bwd(g, oracle_bwd(x, "kda"), "bf16", "kda", what=f"saved kda T={T}")


def test_kda_saved_pair_training_shape_equals_recompute():
    """KDA at the training workload's size (B8 T4096 H16 d128, with du): the training pair
    bit-equals the plain forward and the recomputing backward."""
    from gated_delta_rule_107_b200.inputs import WORKLOADS
    w = WORKLOADS[5]
    x = gen("kda", "bf16", w.B, w.T, w.H, w.dk, w.dv, seed=w.seed, s0_std=w.s0_std, grads=True, du=w.du)
    fwd_ref, bwd_ref = gpu_fwd(x, "kda"), gpu_bwd(x, "kda")
    fwd, g, _ = _save_pair(x, "kda")
    for key in ("o", "u", "S_T"):
        assert torch.equal(fwd[key], fwd_ref[key]), key
    for key, t in g.items():
        if t is not None:
            assert torch.equal(t, bwd_ref[key]), key
