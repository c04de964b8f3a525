"""The single-pass operations around the core (delta_rule_preop / delta_rule_postop and their
backward passes) against the fp64 oracle in oracle/prepost.py, and the pre-operations
feeding the core end to end."""
import numpy as np
import pytest
import torch

from gated_delta_rule_107_b200 import binding
from oracle import prepost as pp
from parity_util import TOL, gpu_fwd, np64, oracle_fwd, rel_err

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def _raw(variant, dtype, B, T, H, d, seed):
    g = torch.Generator().manual_seed(seed)
    r = lambda *s: torch.randn(*s, generator=g).to(DT[dtype]).cuda()  # noqa: E731
    x = {"q": r(B, T, H, d) * 3, "k": r(B, T, H, d) * 3, "b": r(B, T, H)}
    x["a"] = None if variant == "deltanet" else (r(B, T, H, d) if variant == "kda" else r(B, T, H)) - 3.0
    return x


def _check(got, ref, dtype, what):
    err = rel_err(np64(got), ref)
    assert err <= TOL[dtype], f"{what}: {err} (tol {TOL[dtype]})"


@pytest.mark.parametrize("variant", ("deltanet", "gdn", "kda"))
@pytest.mark.parametrize("dtype", ("f32", "bf16"))
@pytest.mark.parametrize("d", (64, 128))
def test_preop_forward_and_backward(variant, dtype, d):
    x = _raw(variant, dtype, 2, 37, 3, d, seed=11 + d)
    q, k, beta, loga = binding.delta_rule_preop(x["q"], x["k"], x["b"], x["a"], variant=variant)
    ref = pp.preop_fwd(np64(x["q"]), np64(x["k"]), np64(x["b"]), np64(x["a"]))
    for key, t in (("q", q), ("k", k), ("beta", beta)):
        _check(t, ref[key], dtype, f"preop {key}")
    if variant == "deltanet":
        assert loga is None
    else:
        _check(loga, ref["loga"], dtype, "preop loga")
    g = torch.Generator().manual_seed(5 + d)
    dq, dk = (torch.randn(q.shape, generator=g).to(q.dtype).cuda() for _ in range(2))
    db = torch.randn(beta.shape, generator=g).to(q.dtype).cuda()
    da = None if loga is None else torch.randn(loga.shape, generator=g).to(q.dtype).cuda()
    gq, gk, gb, ga = binding.delta_rule_preop_bwd(x["q"], x["k"], x["b"], x["a"], dq, dk, db, da, variant=variant)
    torch.cuda.synchronize()
    refb = pp.preop_bwd(np64(x["q"]), np64(x["k"]), np64(x["b"]), np64(x["a"]), np64(dq), np64(dk), np64(db),
                        np64(da))
    for key, t in (("dq", gq), ("dk", gk), ("db", gb)):
        _check(t, refb[key], dtype, f"preop_bwd {key}")
    if variant != "deltanet":
        _check(ga, refb["da"], dtype, "preop_bwd da")


@pytest.mark.parametrize("dtype", ("f32", "bf16"))
@pytest.mark.parametrize("d", (64, 128))
@pytest.mark.parametrize("with_w", (True, False))
def test_postop_forward_and_backward(dtype, d, with_w):
    g = torch.Generator().manual_seed(100 + d)
    B, T, H = 3, 45, 2
    o = (torch.randn(B, T, H, d, generator=g) * 0.3).to(DT[dtype]).cuda()
    gate = torch.randn(B, T, H, d, generator=g).to(DT[dtype]).cuda()
    w = (1.0 + 0.2 * torch.randn(d, generator=g)).cuda() if with_w else None
    dy = torch.randn(B, T, H, d, generator=g).to(DT[dtype]).cuda()
    y = binding.delta_rule_postop(o, gate, w)
    _check(y, pp.postop_fwd(np64(o), np64(gate), np64(w)), dtype, "postop y")
    go, gg, gw = binding.delta_rule_postop_bwd(o, gate, w, dy)
    torch.cuda.synchronize()
    ref = pp.postop_bwd(np64(o), np64(gate), np64(w), np64(dy))
    _check(go, ref["do"], dtype, "postop do")
    _check(gg, ref["dg"], dtype, "postop dg")
    _check(gw, ref["dw"], "f32" if dtype == "f32" else "bf16", "postop dw")
    go2, gg2, gw2 = binding.delta_rule_postop_bwd(o, gate, w, dy)  # deterministic, bit for bit
    torch.cuda.synchronize()
    assert torch.equal(gw, gw2) and torch.equal(go, go2) and torch.equal(gg, gg2)


def test_preop_feeds_the_core():
    """Raw projections -> delta_rule_preop -> delta_rule_fwd equals the oracle run on the
    oracle's own pre-operations (KDA, bf16)."""
    x = _raw("kda", "bf16", 1, 80, 2, 128, seed=7)
    q, k, beta, loga = binding.delta_rule_preop(x["q"], x["k"], x["b"], x["a"], variant="kda")
    g = torch.Generator().manual_seed(8)
    v = torch.randn(1, 80, 2, 128, generator=g).to(torch.bfloat16).cuda()
    got = gpu_fwd({"q": q, "k": k, "v": v, "loga": loga, "beta": beta, "S0": None}, "kda")
    # reference: the oracle's pre-operations rounded to bf16 like the GPU's outputs, then the core oracle
    ref_in = pp.preop_fwd(np64(x["q"]), np64(x["k"]), np64(x["b"]), np64(x["a"]))
    rb = {key: torch.from_numpy(val).to(torch.bfloat16) for key, val in ref_in.items()}
    xo = {"q": rb["q"], "k": rb["k"], "v": v.cpu(), "loga": rb["loga"], "beta": rb["beta"], "S0": None}
    ref = oracle_fwd(xo, "kda")
    for key in ("o", "u", "S_T"):
        assert rel_err(np64(got[key]), ref[key]) <= TOL["bf16"], key


def test_prepost_reject_bad_arguments():
    x = _raw("gdn", "bf16", 1, 4, 1, 128, seed=3)
    out = torch.empty_like(x["q"])
    s = torch.cuda.current_stream().cuda_stream
    p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    base = [p(x["q"]), p(x["k"]), p(x["b"]), p(x["a"]), p(out), p(torch.empty_like(x["k"])),
            p(torch.empty_like(x["b"])), p(torch.empty_like(x["a"]))]
    assert binding.preop_raw(*base, 1, 4, 1, 96, binding.DR_GATED, binding.DR_BF16, s) == binding.DR_ERR_UNSUPPORTED
    assert binding.preop_raw(*base[:3], None, *base[4:], 1, 4, 1, 128, binding.DR_GATED, binding.DR_BF16,
                             s) == binding.DR_ERR_ARG
    assert binding.preop_raw(*base, 1, 4, 1, 128, 9, binding.DR_BF16, s) == binding.DR_ERR_ARG
    assert binding.preop_raw(p(x["q"]) + 2, *base[1:], 1, 4, 1, 128, binding.DR_GATED, binding.DR_BF16,
                             s) == binding.DR_ERR_ALIGN
    assert binding.postop_raw(p(x["q"]), p(x["k"]), None, p(out), 1, 4, 1, 128, binding.DR_BF16, s) == binding.DR_OK
    assert binding.postop_bwd_raw(p(x["q"]), p(x["k"]), None, p(x["q"]), p(out), p(out), None, 1, 4, 1, 128,
                                  binding.DR_BF16, None, 0, s) == binding.DR_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert np.isfinite(np64(out)).all()
