"""The fused forward (delta_rule_fwd_fused): the pre-operation, the forward and the post-operation
in the core's own kernels, against the fp64 oracles chained (oracle/prepost.py's pre-operation,
the core oracle, the post-operation) and against the three separate calls on the GPU."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_107_b200 import binding
from oracle import prepost as pp
from parity_util import TOL, np64, rel_err

pytestmark = pytest.mark.gpu


def _raw(variant, B, T, H, d, seed, s0_std=0.0):
    """Raw projections ~ N(0, 3^2), write-strength logits N(0, 1), forget logits N(0, 1) - 3,
    output gate logits N(0, 1), RMSNorm weight 1 + N(0, 0.2^2)."""
    g = torch.Generator().manual_seed(seed)
    r = lambda *s: torch.randn(*s, generator=g)  # noqa: E731
    x = {"q": r(B, T, H, d) * 3, "k": r(B, T, H, d) * 3, "v": r(B, T, H, d), "b": r(B, T, H),
         "a": None if variant == "deltanet" else r(B, T, H) - 3.0, "go": r(B, T, H, d)}
    x = {k: (None if t is None else t.to(torch.bfloat16).cuda()) for k, t in x.items()}
    x["w"] = (1.0 + 0.2 * r(d)).cuda()
    x["S0"] = (s0_std * r(B, H, d, d)).cuda() if s0_std else None
    return x


def _oracle(x, variant, heads=None):
    sl = (lambda t: t) if heads is None else (lambda t: t[:, :, heads])
    q, k, v, b, go = (np64(sl(x[n])) for n in ("q", "k", "v", "b", "go"))
    a = None if x["a"] is None else np64(sl(x["a"]))
    S0 = None if x["S0"] is None else np64(x["S0"] if heads is None else x["S0"][:, heads])
    pre = pp.preop_fwd(q, k, b, a)
    core = oracle.fwd(pre["q"], pre["k"], v, pre["loga"], pre["beta"], S0, variant=variant)
    core["y"] = pp.postop_fwd(core["o"], go, np64(x["w"]))
    return core


def _fused(x, variant, want_o=True):
    y, o, u, S = binding.delta_rule_fwd_fused(x["q"], x["k"], x["v"], x["a"], x["b"], x["go"], x["w"], S0=x["S0"],
                                              variant=variant, want_o=want_o)
    torch.cuda.synchronize()
    assert binding.sync_status() == binding.DR_OK
    return {"y": y, "o": o, "u": u, "S_T": S}


def _cmp(got, ref, what, heads=None):
    for key in ("y", "o", "u", "S_T"):
        if got[key] is None:
            continue
        g = got[key]
        if heads is not None:
            g = g[:, heads] if key == "S_T" else g[:, :, heads]
        err = rel_err(np64(g), ref[key])
        assert err <= TOL["bf16"], f"{what} {key}: {err}"


@pytest.mark.parametrize("variant", ("gdn", "deltanet"))
@pytest.mark.parametrize("T", (1, 64, 130, 200))
def test_fused_forward_against_chained_oracles(variant, T):
    x = _raw(variant, 2, T, 3, 128, seed=70 + T, s0_std=0.1 if T != 64 else 0.0)
    _cmp(_fused(x, variant), _oracle(x, variant), f"fused {variant} T={T}")


def test_fused_forward_matches_the_three_calls():
    """Against delta_rule_preop, delta_rule_fwd and delta_rule_postop run one after another (the
    fused path keeps the normalised q, k and the gates in fp32, so the two differ by rounding)."""
    x = _raw("gdn", 2, 300, 4, 128, seed=77, s0_std=0.1)
    q, k, beta, loga = binding.delta_rule_preop(x["q"], x["k"], x["b"], x["a"], variant="gdn")
    o, u, S = binding.delta_rule_fwd(q, k, x["v"], loga, beta, x["S0"], variant="gdn")
    y = binding.delta_rule_postop(o, x["go"], x["w"])
    got = _fused(x, "gdn")
    for key, ref in (("y", y), ("o", o), ("u", u), ("S_T", S)):
        err = rel_err(np64(got[key]), np64(ref))
        assert err <= TOL["bf16"], f"{key}: {err}"


def test_fused_forward_without_optional_outputs():
    x = _raw("gdn", 1, 150, 2, 128, seed=78)
    y, o, u, S = binding.delta_rule_fwd_fused(x["q"], x["k"], x["v"], x["a"], x["b"], x["go"], x["w"], variant="gdn",
                                              want_o=False, want_u=False, want_state=False)
    torch.cuda.synchronize()
    assert o is None and u is None and S is None
    err = rel_err(np64(y), _oracle(x, "gdn")["y"])
    assert err <= TOL["bf16"], err


def test_fused_forward_headline_shape_sampled_heads():
    """B8 T4096 H8 d128 (the headline shape); heads are independent, so the oracle runs two."""
    x = _raw("gdn", 8, 4096, 8, 128, seed=79)
    got = _fused(x, "gdn")
    _cmp(got, _oracle(x, "gdn", heads=[1, 6]), "fused headline", heads=[1, 6])
    assert torch.isfinite(got["y"]).all()


def test_fused_forward_serves_only_its_configurations():
    x = _raw("gdn", 1, 8, 1, 64, seed=80)
    p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    s = torch.cuda.current_stream().cuda_stream
    args = (p(x["q"]), p(x["k"]), p(x["v"]), p(x["a"]), p(x["b"]), None, p(x["go"]), p(x["w"]), p(x["v"]), None,
            None, None)
    for variant, d, dt in ((binding.DR_KDA, 128, binding.DR_BF16), (binding.DR_GATED, 64, binding.DR_BF16),
                           (binding.DR_GATED, 128, binding.DR_F32)):
        assert binding.fwd_fused_raw(*args, 1, 8, 1, d, d, variant, 64, dt, None, 0, s) == binding.DR_ERR_UNSUPPORTED
