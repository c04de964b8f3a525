"""Seeded synthetic inputs for the gated delta rule.

This module only draws random numbers in the shapes and distributions of the
workloads; it holds none of the recurrence's arithmetic.  Both the CUDA path and
the CPU oracle consume exactly the values it returns (the oracle widens the
stored I/O-dtype values to fp64).

Distributions:
  * q, k ~ N(0, 1), then L2-normalised per (token, head) -- the Kimi Delta
    Attention page ("线性注意力架构演进与Kimi Delta Attention创新实践") applies an L2
    norm to q and k before the core (sections 2.1 and 7.1).
  * v ~ N(0, 1).
  * beta = sigmoid(N(0, 1)).
  * log alpha = -softplus(N(-3, 1)), i.e. log(sigmoid(x)) with x ~ N(-3, 1): the
    forget-gate bias of -3 from the same page, section 7.1.  One value per
    (token, head) for Gated DeltaNet, one per key channel for KDA, none for
    DeltaNet.
  * S0 ~ N(0, s0_std) when s0_std > 0, else absent (zero state).
  * upstream gradients dO, du, dS_T ~ N(0, 1) when requested.

Draw order is fixed (q, k, v, log alpha, beta, S0, dO, du, dS_T) from one CPU
``torch.Generator`` seeded with ``seed``, so a workload is reproducible on any
machine; values are drawn in fp32 and cast to the I/O dtype.
"""
from __future__ import annotations

import dataclasses

import torch

DELTANET, GATED, KDA = 0, 1, 2
VARIANT_NAMES = {DELTANET: "deltanet", GATED: "gdn", KDA: "kda"}
VARIANT_IDS = {"deltanet": DELTANET, "gdn": GATED, "gated": GATED, "kda": KDA}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    variant: int
    dtype: str  # "f32" or "bf16"
    B: int
    T: int
    H: int
    dk: int
    dv: int
    s0_std: float = 0.0
    backward: bool = False
    du: bool = False
    seed: int = 0


# The five benchmark workloads (sizes and distributions as stated for each).
WORKLOADS = {
    1: Workload("deltanet_fwd_f32_B1_T256_H2_d64", DELTANET, "f32", 1, 256, 2, 64, 64, seed=1001),
    2: Workload("gdn_bf16_B8_T4096_H8_d128", GATED, "bf16", 8, 4096, 8, 128, 128, seed=1002),
    3: Workload("kda_fwd_bf16_B4_T16384_H8_d128_s0", KDA, "bf16", 4, 16384, 8, 128, 128, s0_std=0.02, seed=1003),
    4: Workload("gdn_fwdbwd_bf16_B1_T32768_H16_d128", GATED, "bf16", 1, 32768, 16, 128, 128, backward=True,
                seed=1004),
    5: Workload("kda_fwdbwd_bf16_B8_T4096_H16_d128_du", KDA, "bf16", 8, 4096, 16, 128, 128, backward=True, du=True,
                seed=1005),
}

TORCH_DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


def _l2n(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-6)


def make_inputs(variant, dtype: str, B: int, T: int, H: int, dk: int, dv: int, seed: int, s0_std: float = 0.0,
                grads: bool = False, du: bool = True, device="cpu") -> dict:
    """Draw one workload's tensors.  Returns a dict of tensors on ``device``.

    Keys: q, k, v, loga (None for deltanet), beta, S0 (None unless s0_std > 0),
    and with ``grads``: dO, du (None unless ``du``), dS_T.
    Per-token tensors have the I/O dtype; S0 / dS_T are fp32.
    """
    var = VARIANT_IDS[variant] if isinstance(variant, str) else int(variant)
    td = TORCH_DTYPES[dtype]
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed))

    def normal(shape, mean=0.0, std=1.0):
        x = torch.empty(shape, dtype=torch.float32)
        x.normal_(mean=mean, std=std, generator=gen)
        return x

    out = {}
    out["q"] = _l2n(normal((B, T, H, dk))).to(td)
    out["k"] = _l2n(normal((B, T, H, dk))).to(td)
    out["v"] = normal((B, T, H, dv)).to(td)
    if var == DELTANET:
        out["loga"] = None
    else:
        gshape = (B, T, H, dk) if var == KDA else (B, T, H)
        out["loga"] = (-torch.nn.functional.softplus(normal(gshape, mean=-3.0))).to(td)
    out["beta"] = torch.sigmoid(normal((B, T, H))).to(td)
    out["S0"] = normal((B, H, dk, dv), std=s0_std) if s0_std > 0 else None
    if grads:
        out["dO"] = normal((B, T, H, dv)).to(td)
        out["du"] = normal((B, T, H, dv)).to(td) if du else None
        out["dS_T"] = normal((B, H, dk, dv))
    if device != "cpu":
        out = {key: (val.to(device) if val is not None else None) for key, val in out.items()}
    return out


def workload_inputs(wid: int, device="cpu", **overrides) -> tuple[Workload, dict]:
    """Inputs of workload ``wid`` (optionally with fields replaced, e.g. T=128)."""
    w = dataclasses.replace(WORKLOADS[wid], **overrides) if overrides else WORKLOADS[wid]
    t = make_inputs(w.variant, w.dtype, w.B, w.T, w.H, w.dk, w.dv, w.seed, s0_std=w.s0_std, grads=w.backward,
                    du=w.du, device=device)
    return w, t
