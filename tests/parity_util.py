"""Helpers shared by the GPU parity tests: run both sides on the same inputs, compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from gated_delta_rule_107_b200 import binding
from gated_delta_rule_107_b200.inputs import VARIANT_NAMES, make_inputs

# max|gpu - oracle| / max|oracle| per output tensor: the stated bar for fp32 I/O and for
# bf16 I/O with an fp32 state.
TOL = {"f32": 1e-4, "bf16": 2e-2}


def rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = float(np.max(np.abs(ref))) if ref.size else 0.0
    num = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    if den == 0.0:
        return num
    return num / den


def np64(t):
    return None if t is None else t.detach().to("cpu").double().numpy()


def gen(variant, dtype, B, T, H, dk, dv, seed, s0_std=0.0, grads=False, du=True):
    return make_inputs(variant, dtype, B, T, H, dk, dv, seed, s0_std=s0_std, grads=grads, du=du, device="cuda")


def heads_slice(x, heads):
    """Restrict every [B,T,H,...] / [B,H,...] tensor to the given head indices (heads are independent)."""
    out = {}
    for key, t in x.items():
        if t is None:
            out[key] = None
        elif key in ("S0", "dS_T"):
            out[key] = t[:, heads]
        else:
            out[key] = t[:, :, heads]
    return out


def gpu_fwd(x, variant, chunk=64):
    o, u, S = binding.delta_rule_fwd(x["q"], x["k"], x["v"], x["loga"], x["beta"], x["S0"], variant=variant,
                                     chunk=chunk)
    torch.cuda.synchronize()
    assert binding.sync_status() == binding.DR_OK
    return {"o": o, "u": u, "S_T": S}


def gpu_bwd(x, variant, chunk=64):
    g = binding.delta_rule_bwd(x["q"], x["k"], x["v"], x["loga"], x["beta"], x["S0"], x["dO"], x.get("du"),
                               x.get("dS_T"), variant=variant, chunk=chunk)
    torch.cuda.synchronize()
    assert binding.sync_status() == binding.DR_OK
    return g


def oracle_fwd(x, variant, heads=None):
    if heads is not None:
        x = heads_slice(x, heads)
    return oracle.fwd(*(np64(x[key]) for key in ("q", "k", "v", "loga", "beta", "S0")), variant=variant)


def oracle_bwd(x, variant, heads=None):
    if heads is not None:
        x = heads_slice(x, heads)
    return oracle.bwd(*(np64(x[key]) for key in ("q", "k", "v", "loga", "beta", "S0")),
                      dO=np64(x["dO"]), du=np64(x.get("du")), dS_T=np64(x.get("dS_T")), variant=variant)


def compare_fwd(got, ref, dtype, heads=None, what=""):
    errs = {}
    for key in ("o", "u", "S_T"):
        g = got[key]
        if heads is not None:
            g = g[:, heads] if key == "S_T" else g[:, :, heads]
        errs[key] = rel_err(np64(g), ref[key])
    bad = {k: v for k, v in errs.items() if not v <= TOL[dtype]}
    assert not bad, f"{what} forward parity {errs} (tol {TOL[dtype]})"
    return errs


GRAD_KEYS = (("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("dbeta", "dbeta"), ("dS0", "dS0"), ("dalpha", "dloga"))


def compare_bwd(got, ref, dtype, variant, heads=None, what=""):
    errs = {}
    for gk, rk in GRAD_KEYS:
        if gk == "dalpha" and VARIANT_NAMES.get(variant, variant) == "deltanet":
            continue
        g = got[gk]
        if heads is not None:
            g = g[:, heads] if gk == "dS0" else g[:, :, heads]
        errs[gk] = rel_err(np64(g), ref[rk])
    bad = {k: v for k, v in errs.items() if not v <= TOL[dtype]}
    assert not bad, f"{what} backward parity {errs} (tol {TOL[dtype]})"
    return errs
