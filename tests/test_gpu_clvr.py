"""Cross-layer value routing (delta_rule_clvr / _bwd) against the fp64 oracle in oracle/clvr.py:
the zero-initialised projection leaves the hidden stream bit for bit, the in-place residual
add, the core's own write values routed, the headline shape on sampled rows, and argument
checks."""
import numpy as np
import pytest
import torch

from gated_delta_rule_107_b200 import binding
from oracle import clvr as cl
from parity_util import TOL, gen, gpu_fwd, np64, oracle_fwd, rel_err

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def _check(got, ref, tol, what):
    err = rel_err(got if isinstance(got, np.ndarray) else np64(got), ref)
    assert err <= tol, f"{what}: {err} (tol {tol})"


@pytest.mark.parametrize("dtype", ("f32", "bf16"))
# (2, 200, 3, 128, 384): M = 400 and N = 384, so in the last row and column blocks of 256 the
# first CTA of a pair holds 128 valid rows / columns and the second a part (rows 384-399) or none
@pytest.mark.parametrize("shape", ((1, 5, 2, 64, 128), (2, 150, 8, 128, 1024), (3, 37, 4, 64, 40),
                                   (2, 200, 3, 128, 384)))
def test_forward_and_backward(dtype, shape):
    B, T, H, dv, N = shape
    g = torch.Generator().manual_seed(B * 1000 + T)
    u = (0.3 * torch.randn(B, T, H, dv, generator=g)).to(DT[dtype]).cuda()
    W = (0.05 * torch.randn(H * dv, N, generator=g)).to(DT[dtype]).cuda()
    h = torch.randn(B, T, N, generator=g).to(DT[dtype]).cuda()
    dh = torch.randn(B, T, N, generator=g).to(DT[dtype]).cuda()
    out = binding.delta_rule_clvr(u, W, h)
    du, dW = binding.delta_rule_clvr_bwd(u, W, dh)
    torch.cuda.synchronize()
    _check(out.reshape(B * T, N), cl.clvr_fwd(np64(u), np64(W), np64(h)), TOL[dtype], "h_out")
    ref = cl.clvr_bwd(np64(u), np64(W), np64(dh))
    _check(du.reshape(B * T, H * dv), ref["du"], TOL[dtype], "du")
    _check(dW, ref["dW"], TOL[dtype], "dW")
    # no residual: u W alone
    _check(binding.delta_rule_clvr(u, W), cl.clvr_fwd(np64(u), np64(W)), TOL[dtype], "u W")


def test_zero_projection_is_identity_and_in_place():
    g = torch.Generator().manual_seed(4)
    u = torch.randn(2, 64, 8, 128, generator=g).to(torch.bfloat16).cuda()
    h = torch.randn(2, 64, 1024, generator=g).to(torch.bfloat16).cuda()
    W0 = torch.zeros(1024, 1024, dtype=torch.bfloat16, device="cuda")
    out = binding.delta_rule_clvr(u, W0, h)
    torch.cuda.synchronize()
    assert torch.equal(out, h)  # the zero-initialised routing changes nothing
    W = (0.05 * torch.randn(1024, 1024, generator=g)).to(torch.bfloat16).cuda()
    ref = cl.clvr_fwd(np64(u), np64(W), np64(h))
    binding.delta_rule_clvr(u, W, h, out=h)  # in place
    torch.cuda.synchronize()
    _check(h.reshape(128, 1024), ref, TOL["bf16"], "in place")


def test_routes_the_cores_write_values():
    x = gen("gdn", "bf16", 1, 130, 2, 128, 128, seed=17)
    u = gpu_fwd(x, "gdn")["u"]
    g = torch.Generator().manual_seed(3)
    W = (0.05 * torch.randn(256, 256, generator=g)).to(torch.bfloat16).cuda()
    h = torch.randn(1, 130, 256, generator=g).to(torch.bfloat16).cuda()
    out = binding.delta_rule_clvr(u, W, h)
    torch.cuda.synchronize()
    ref_u = oracle_fwd(x, "gdn")["u"]
    _check(out.reshape(130, 256), cl.clvr_fwd(ref_u, np64(W), np64(h)), TOL["bf16"], "core u routed")


def test_headline_shape_sampled_rows():
    """B8 T4096, H8 dv128 write values into a 1024-wide hidden stream (bf16); rows are
    independent, so the oracle checks a sample of 512 of them."""
    B, T, H, dv, N = 8, 4096, 8, 128, 1024
    g = torch.Generator().manual_seed(8)
    u = (0.3 * torch.randn(B, T, H, dv, generator=g)).to(torch.bfloat16).cuda()
    W = (0.05 * torch.randn(H * dv, N, generator=g)).to(torch.bfloat16).cuda()
    h = torch.randn(B, T, N, generator=g).to(torch.bfloat16).cuda()
    dh = torch.randn(B, T, N, generator=g).to(torch.bfloat16).cuda()
    out = binding.delta_rule_clvr(u, W, h)
    du, dW = binding.delta_rule_clvr_bwd(u, W, dh)
    torch.cuda.synchronize()
    rows = np.random.default_rng(0).choice(B * T, 512, replace=False)
    U, Hh, dH = np64(u).reshape(B * T, H * dv), np64(h).reshape(B * T, N), np64(dh).reshape(B * T, N)
    _check(np64(out).reshape(B * T, N)[rows], cl.clvr_fwd(U[rows], np64(W), Hh[rows]), TOL["bf16"], "h_out")
    _check(np64(du).reshape(B * T, H * dv)[rows], cl.clvr_bwd(U[rows], np64(W), dH[rows])["du"], TOL["bf16"], "du")
    # dW sums over every row: check it whole
    _check(dW, cl.clvr_bwd(U, np64(W), dH)["dW"], TOL["bf16"], "dW")


def test_clvr_rejects_bad_arguments():
    u = torch.randn(4, 64, dtype=torch.bfloat16, device="cuda")
    W = torch.randn(64, 64, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(4, 64, dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    need = binding.load().delta_rule_clvr_workspace_size()
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    P = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    assert binding.clvr_raw(P(u), P(W), None, P(out), 4, 60, 64, binding.DR_BF16, P(ws), need, s) == \
        binding.DR_ERR_UNSUPPORTED
    assert binding.clvr_raw(P(u), P(W), None, P(out), 4, 64, 64, binding.DR_BF16, None, 0, s) == \
        binding.DR_ERR_WORKSPACE
    assert binding.clvr_raw(P(u) + 2, P(W), None, P(out), 4, 64, 64, binding.DR_BF16, P(ws), need, s) == \
        binding.DR_ERR_ALIGN
    assert binding.clvr_raw(None, P(W), None, P(out), 4, 64, 64, binding.DR_BF16, P(ws), need, s) == binding.DR_ERR_ARG
    dW = torch.full((64, 64), float("nan"), device="cuda")
    assert binding.clvr_bwd_raw(P(u), P(W), P(out), None, P(dW), 0, 64, 64, binding.DR_BF16, None, 0, s) == \
        binding.DR_OK
    torch.cuda.synchronize()
    assert torch.equal(dW, torch.zeros_like(dW))  # no tokens: an empty sum


def test_dw_split_reduction_is_deterministic():
    """dW's reduction over the tokens runs in slices whose partials are added in a fixed order:
    two calls return the same bits."""
    g = torch.Generator().manual_seed(9)
    u = (0.3 * torch.randn(4, 1000, 4, 128, generator=g)).to(torch.bfloat16).cuda()
    W = (0.05 * torch.randn(512, 768, generator=g)).to(torch.bfloat16).cuda()
    dh = torch.randn(4, 1000, 768, generator=g).to(torch.bfloat16).cuda()
    _, dW1 = binding.delta_rule_clvr_bwd(u, W, dh)
    _, dW2 = binding.delta_rule_clvr_bwd(u, W, dh)
    torch.cuda.synchronize()
    assert torch.equal(dW1, dW2)
    _check(dW1, cl.clvr_bwd(np64(u), np64(W), np64(dh))["dW"], TOL["bf16"], "dW")
