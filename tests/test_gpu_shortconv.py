"""The kernel-4 depthwise causal short convolution (delta_rule_shortconv / _bwd) against the fp64
oracle in oracle/shortconv.py: ragged token counts around the kernels' token blocks, with and
without the three-token cache, the stream split across calls, a deterministic dw, the full-size
q stream of the headline shape, and argument checks."""
import numpy as np
import pytest
import torch

from gated_delta_rule_107_b200 import binding
from oracle import shortconv as sc
from parity_util import TOL, np64, rel_err

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def _inputs(dtype, B, T, D, seed, prev=True):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(B, T, D, generator=g).to(DT[dtype]).cuda()
    w = (0.5 * torch.randn(D, 4, generator=g)).cuda()
    p = torch.randn(B, 3, D, generator=g).to(DT[dtype]).cuda() if prev else None
    dy = torch.randn(B, T, D, generator=g).to(DT[dtype]).cuda()
    return x, w, p, dy


def _check(got, ref, tol, what):
    err = rel_err(got if isinstance(got, np.ndarray) else np64(got), ref)
    assert err <= tol, f"{what}: {err} (tol {tol})"


@pytest.mark.parametrize("dtype", ("f32", "bf16"))
@pytest.mark.parametrize("T", (0, 1, 2, 5, 16, 17, 63, 64, 65, 130))
@pytest.mark.parametrize("prev", (False, True))
def test_forward_and_backward(dtype, T, prev):
    B, D = 2, 40
    x, w, p, dy = _inputs(dtype, B, T, D, seed=300 + T, prev=prev)
    y, cache = binding.delta_rule_shortconv(x, w, p, want_cache=True)
    dx, dw, dprev = binding.delta_rule_shortconv_bwd(x, w, dy, p, want_dprev=True)
    torch.cuda.synchronize()
    ry, rcache = sc.shortconv_fwd(np64(x), np64(w), np64(p))
    rb = sc.shortconv_bwd(np64(x), np64(w), np64(dy), np64(p))
    if T:
        _check(y, ry, TOL[dtype], "y")
        _check(dx, rb["dx"], TOL[dtype], "dx")
    assert np.array_equal(np64(cache), rcache)  # a copy of input tokens: exact
    _check(dw, rb["dw"], TOL["f32"], "dw")      # fp32 sums of products of I/O values
    _check(dprev, rb["dx_prev"], TOL[dtype], "dx_prev")


def test_stream_split_is_exact_and_dw_deterministic():
    B, T, D = 3, 150, 64
    x, w, _, dy = _inputs("bf16", B, T, D, seed=11, prev=False)
    whole, cache = binding.delta_rule_shortconv(x, w, want_cache=True)
    parts, c = [], None
    for a, b in ((0, 1), (1, 3), (3, 40), (40, 150)):
        y, c = binding.delta_rule_shortconv(x[:, a:b].contiguous(), w, c, want_cache=True)
        parts.append(y)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(parts, dim=1), whole) and torch.equal(c, cache)
    _, dw1, _ = binding.delta_rule_shortconv_bwd(x, w, dy)
    _, dw2, _ = binding.delta_rule_shortconv_bwd(x, w, dy)
    torch.cuda.synchronize()
    assert torch.equal(dw1, dw2)


def test_head_layout_and_full_size_q_stream():
    """[B, T, H, d] input at the headline shape (B8 T4096 H8 d128, bf16): one D = 1024 stream."""
    B, T, H, d = 8, 4096, 8, 128
    g = torch.Generator().manual_seed(5)
    x = torch.randn(B, T, H, d, generator=g).to(torch.bfloat16).cuda()
    w = (0.5 * torch.randn(H * d, 4, generator=g)).cuda()
    dy = torch.randn(B, T, H, d, generator=g).to(torch.bfloat16).cuda()
    y = binding.delta_rule_shortconv(x, w)
    dx, dw, _ = binding.delta_rule_shortconv_bwd(x, w, dy)
    torch.cuda.synchronize()
    xs, dys = np64(x).reshape(B, T, H * d), np64(dy).reshape(B, T, H * d)
    ry, _ = sc.shortconv_fwd(xs, np64(w))
    rb = sc.shortconv_bwd(xs, np64(w), dys)
    _check(y.reshape(B, T, H * d), ry, TOL["bf16"], "y")
    _check(dx.reshape(B, T, H * d), rb["dx"], TOL["bf16"], "dx")
    _check(dw, rb["dw"], TOL["f32"], "dw")


def test_shortconv_rejects_bad_arguments():
    x, w, p, dy = _inputs("bf16", 1, 8, 64, seed=3)
    y = torch.empty_like(x)
    s = torch.cuda.current_stream().cuda_stream
    P = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    assert binding.shortconv_raw(P(x), P(w), None, P(y), None, 1, 8, 60, binding.DR_BF16, s) == \
        binding.DR_ERR_UNSUPPORTED
    assert binding.shortconv_raw(P(x), None, None, P(y), None, 1, 8, 64, binding.DR_BF16, s) == binding.DR_ERR_ARG
    assert binding.shortconv_raw(P(x) + 2, P(w), None, P(y), None, 1, 8, 64, binding.DR_BF16, s) == \
        binding.DR_ERR_ALIGN
    assert binding.shortconv_raw(P(x), P(w), None, P(y), None, 1, 8, 64, 5, s) == binding.DR_ERR_ARG
    dx, dw = torch.empty_like(x), torch.empty(64, 4, device="cuda")
    assert binding.shortconv_bwd_raw(P(x), P(w), None, P(dy), P(dx), P(dw), None, 1, 8, 64, binding.DR_BF16, None, 0,
                                     s) == binding.DR_ERR_WORKSPACE
    # no dw: no workspace needed
    assert binding.shortconv_bwd_raw(P(x), P(w), None, P(dy), P(dx), None, None, 1, 8, 64, binding.DR_BF16, None, 0,
                                     s) == binding.DR_OK
    # T = 0: the cache passes through
    c = torch.empty_like(p)
    assert binding.shortconv_raw(None, P(w), P(p), None, P(c), 1, 0, 64, binding.DR_BF16, s) == binding.DR_OK
    torch.cuda.synchronize()
    assert torch.equal(c, p)
