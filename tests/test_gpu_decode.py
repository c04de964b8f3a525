"""The recurrent form for decoding (delta_rule_decode) against the fp64 oracle.

The decode entry point steps the same recurrence token by token, so its reference is the
oracle's token-by-token forward from the same initial state; it must also agree with the
chunked forward on the same tokens, and splitting the tokens into several decoding calls
that hand the state on must give the same result bit for bit.
"""
import pytest
import torch

from gated_delta_rule_107_b200 import binding
from parity_util import compare_fwd, gen, gpu_fwd, np64, oracle_fwd, rel_err, TOL

pytestmark = pytest.mark.gpu


def _decode(x, variant, S=None, inplace=False):
    S = x["S0"] if S is None else S
    o, u, S_out = binding.delta_rule_decode(x["q"], x["k"], x["v"], x["loga"], x["beta"], S, variant=variant,
                                            inplace=inplace)
    torch.cuda.synchronize()
    assert binding.sync_status() == binding.DR_OK
    return {"o": o, "u": u, "S_T": S_out}


@pytest.mark.parametrize("variant", ("deltanet", "gdn", "kda"))
@pytest.mark.parametrize("dtype", ("f32", "bf16"))
@pytest.mark.parametrize("T,d", ((1, 128), (3, 64), (17, 128), (40, 64)))
def test_decode_matches_oracle(variant, dtype, T, d):
    x = gen(variant, dtype, 2, T, 3, d, d, seed=71 + T + d, s0_std=0.05)
    compare_fwd(_decode(x, variant), oracle_fwd(x, variant), dtype, what=f"decode {variant} {dtype} T={T}")


@pytest.mark.parametrize("variant", ("gdn", "kda"))
def test_decode_mixed_key_value_widths(variant):
    x = gen(variant, "bf16", 1, 5, 2, 128, 64, seed=83, s0_std=0.05)
    compare_fwd(_decode(x, variant), oracle_fwd(x, variant), "bf16", what=f"decode {variant} dk128 dv64")
    x = gen(variant, "bf16", 1, 5, 2, 64, 128, seed=84, s0_std=0.05)
    compare_fwd(_decode(x, variant), oracle_fwd(x, variant), "bf16", what=f"decode {variant} dk64 dv128")


def test_decode_in_place_and_split_calls_are_exact():
    x = gen("gdn", "bf16", 3, 21, 4, 128, 128, seed=91, s0_std=0.05)
    whole = _decode(x, "gdn")
    S = x["S0"].clone()
    parts = []
    for a, b in ((0, 1), (1, 9), (9, 21)):  # three decoding calls, the state updated in place
        xs = {k: (t[:, a:b].contiguous() if k != "S0" and t is not None else t) for k, t in x.items()}
        parts.append(_decode(xs, "gdn", S=S, inplace=True))
    assert torch.equal(S, whole["S_T"])
    for key in ("o", "u"):
        assert torch.equal(torch.cat([p[key] for p in parts], dim=1), whole[key]), key


def test_decode_agrees_with_chunked_forward():
    x = gen("kda", "bf16", 2, 70, 2, 128, 128, seed=93, s0_std=0.05)
    dec, chk = _decode(x, "kda"), gpu_fwd(x, "kda")
    for key in ("o", "u", "S_T"):
        assert rel_err(np64(dec[key]), np64(chk[key])) <= TOL["bf16"], key


def test_decode_zero_state_and_empty_sequence():
    x = gen("gdn", "f32", 1, 4, 2, 64, 64, seed=95)
    assert x["S0"] is None  # no initial state: decoding starts from zero
    compare_fwd(_decode(x, "gdn"), oracle_fwd(x, "gdn"), "f32", what="decode from a zero state")
    S = torch.randn(1, 2, 64, 64, device="cuda")
    S_out = torch.full_like(S, float("nan"))
    e = x["q"][:, :0]
    rc = binding.decode_raw(e.data_ptr(), e.data_ptr(), e.data_ptr(), x["loga"].data_ptr(), x["beta"].data_ptr(),
                            S.data_ptr(), S_out.data_ptr(), e.data_ptr(), None, 1, 0, 2, 64, 64, binding.DR_GATED,
                            binding.DR_F32, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert rc == binding.DR_OK and torch.equal(S_out, S)


def test_decode_rejects_bad_arguments():
    x = gen("gdn", "bf16", 1, 2, 1, 128, 128, seed=97)
    p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    o = torch.empty_like(x["v"])
    stream = torch.cuda.current_stream().cuda_stream

    def call(q=p(x["q"]), alpha=p(x["loga"]), dk=128, variant=binding.DR_GATED, out=p(o)):
        return binding.decode_raw(q, p(x["k"]), p(x["v"]), alpha, p(x["beta"]), None, None, out, None, 1, 2, 1, dk,
                                  128, variant, binding.DR_BF16, stream)

    assert call(dk=96) == binding.DR_ERR_UNSUPPORTED
    assert call(variant=7) == binding.DR_ERR_ARG
    assert call(alpha=None) == binding.DR_ERR_ARG
    assert call(out=None) == binding.DR_ERR_ARG
    assert call(q=p(x["q"]) + 2) == binding.DR_ERR_ALIGN
    assert call() == binding.DR_OK
    torch.cuda.synchronize()
