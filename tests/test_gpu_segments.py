"""Long sequences with few (b, h) pairs (Gated DeltaNet, DeltaNet, KDA on the tensor-core path):
the library cuts each sequence's chunk range into four segments, so that the prep of one
segment runs beside the forward chain of the one before and the gradient kernel of one beside
the reverse chain of the one before, with the states at the cuts kept in fp32.  The timed entry
points run one launch per kernel over the whole range, so both must give the same results bit
for bit, and those match the fp64 oracle."""
import pytest
import torch

from gated_delta_rule_107_b200 import binding
from parity_util import compare_bwd, compare_fwd, gen, gpu_bwd, gpu_fwd, oracle_bwd, oracle_fwd

pytestmark = pytest.mark.gpu

C, DT = 64, binding.DR_BF16


def _saved_pair(x, variant, timed):
    B, T, H, dk = x["q"].shape
    dv = x["v"].shape[-1]
    var = binding.VARIANTS[variant]
    p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    o, u = torch.empty_like(x["v"]), torch.empty_like(x["v"])
    S_T = torch.empty(B, H, dk, dv, dtype=torch.float32, device="cuda")
    g = {"dq": torch.empty_like(x["q"]), "dk": torch.empty_like(x["k"]), "dv": torch.empty_like(x["v"]),
         "dalpha": torch.empty_like(x["loga"]) if variant != "deltanet" else None,
         "dbeta": torch.empty_like(x["beta"]),
         "dS0": torch.empty(B, H, dk, dv, dtype=torch.float32, device="cuda")}
    svb = binding.saved_size(B, T, H, dk, dv, var, C, DT)
    saved = torch.empty(svb, dtype=torch.uint8, device="cuda")
    nws = max(binding.workspace_size(B, T, H, dk, dv, var, C, DT, kind) for kind in (2, 3))
    ws = torch.empty(max(nws, 256), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    fa = (p(x["q"]), p(x["k"]), p(x["v"]), p(x["loga"]), p(x["beta"]), p(x["S0"]), p(o), p(u), p(S_T),
          B, T, H, dk, dv, var, C, DT)
    ba = (p(x["q"]), p(x["k"]), p(x["v"]), p(x["loga"]), p(x["beta"]), p(x["S0"]), p(x["dO"]), p(x.get("du")),
          p(x.get("dS_T")), p(g["dq"]), p(g["dk"]), p(g["dv"]), p(g["dalpha"]), p(g["dbeta"]), p(g["dS0"]),
          B, T, H, dk, dv, var, C, DT)
    sv, wsa = (p(saved), svb), (p(ws), ws.numel(), stream)
    if timed:
        fe = [torch.cuda.Event(enable_timing=True) for _ in range(len(binding.launches(B, T, H, dk, dv, var, C, DT, 2)) + 1)]
        be = [torch.cuda.Event(enable_timing=True) for _ in range(len(binding.launches(B, T, H, dk, dv, var, C, DT, 3)) + 1)]
        for e in fe + be:  # torch creates the CUDA event handle on first record
            e.record()
        torch.cuda.synchronize()
        rc1 = binding.fwd_save_timed_raw(*fa, *sv, *wsa, binding.event_array(fe), len(fe))
        rc2 = binding.bwd_saved_timed_raw(*ba, *sv, *wsa, binding.event_array(be), len(be))
    else:
        rc1 = binding.fwd_save_raw(*fa, *sv, *wsa)
        rc2 = binding.bwd_saved_raw(*ba, *sv, *wsa)
    assert rc1 == binding.DR_OK and rc2 == binding.DR_OK, (rc1, rc2)
    torch.cuda.synchronize()
    assert binding.sync_status() == binding.DR_OK
    return {"o": o, "u": u, "S_T": S_T}, {k: v for k, v in g.items() if v is not None}


# (variant, B, T, H, du, S0 std, fast): 8 or 12 chains with 65 or 33 chunks (segments of 16-17
# or 8-9); fast: KDA channels whose gates fall by 12 nats a token in one sequence, so that
# some chunks go to the CUDA-core gradient kernel after the segments
@pytest.mark.parametrize("variant,B,T,H,du,s0,fast", (("gdn", 1, 4133, 4, True, 0.1, False),
                                                      ("deltanet", 2, 2100, 3, False, 0.0, False),
                                                      ("kda", 1, 2100, 4, True, 0.1, False),
                                                      ("kda", 2, 2100, 2, True, 0.0, True)))
def test_segments_equal_whole_range_and_oracle(variant, B, T, H, du, s0, fast):
    x = gen(variant, "bf16", B, T, H, 128, 128, seed=71 + T, s0_std=s0, grads=True, du=du)
    if fast:
        x["loga"][0, :, :, :4] = -12.0
        x["loga"][..., 4:8] = -3.0
    f_seg, g_seg = _saved_pair(x, variant, timed=False)
    f_one, g_one = _saved_pair(x, variant, timed=True)
    for key in f_one:
        assert torch.equal(f_seg[key], f_one[key]), key
    for key in g_one:
        assert torch.equal(g_seg[key], g_one[key]), key
    # the plain forward and the recomputing backward, cut into segments the same way
    f_plain, g_plain = gpu_fwd(x, variant), gpu_bwd(x, variant)
    for key in f_one:
        assert torch.equal(f_plain[key], f_one[key]), key
    for key in g_one:
        assert torch.equal(g_plain[key], g_one[key]), key
    compare_fwd(f_seg, oracle_fwd(x, variant), "bf16", what=f"segmented {variant} T={T}")
    compare_bwd(g_seg, oracle_bwd(x, variant), "bf16", variant, what=f"segmented {variant} T={T}")


def test_plain_launch_counts():
    # segmented: each of the forward's two kernels and the backward's two once per segment
    args = (1, 4133, 4, 128, 128, binding.VARIANTS["gdn"], C, DT)
    assert len(binding.launches(*args, 2)) == 2 and binding.plain_launches(*args, 2) == 8
    assert len(binding.launches(*args, 3)) == 2 and binding.plain_launches(*args, 3) == 8
    assert binding.plain_launches(*args, 1) == 4 - 2 + 8  # the recompute's prep and chain once
    # the headline shape (128 chain CTAs) runs whole: the same count as the timed form
    args = (8, 4096, 8, 128, 128, binding.VARIANTS["gdn"], C, DT)
    for kind in range(4):
        assert binding.plain_launches(*args, kind) == len(binding.launches(*args, kind))
