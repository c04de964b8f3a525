"""Pins that tie the fp64 oracle to facts fixed outside the oracle itself.

Each ``pin_*`` takes a loaded oracle library handle (``oracle.load_library()`` or
a deliberately broken build of it) and raises ``AssertionError`` on failure.
``test_oracle_pins.py`` runs them on the real oracle; ``test_oracle_mutants.py``
runs them on copies of the oracle with planted mistakes and requires that every
mistake is caught by at least one pin.

Sources of the facts:
  * The state update of the Kimi Delta Attention page
    ("线性注意力架构演进与Kimi Delta Attention创新实践", section 2.1) -- the
    hand-worked example in tests/golden/, the T=1 and matrix-product forms.
  * The variant nesting (explainer "线性注意力架构：机制、权衡与跨层路由", core
    method 1; ETH news article, section 二): channel gates that coincide reduce
    KDA to Gated DeltaNet; alpha == 1 is DeltaNet.
  * The delta rule writes only the correction (ETH news article, section 二:
    DeltaNet "only records the patch"), so a unit key with beta = 1 recalls its
    value exactly and orthonormal keys never interfere.
  * Linear algebra: the chunked (UT / WY) solve, linearity in (S0, V), the
    split-sequence identity, the state reconstruction from u, the adjoint
    identity and finite differences.
"""
from __future__ import annotations

import json
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "hand_example_d2_T2.json")
VARS = ("deltanet", "gdn", "kda")


def rand_inputs(rng, B, T, H, dk, dv, variant, s0=True, gate_scale=1.0, unit_keys=True):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    if unit_keys:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    if variant == "kda":
        loga = -np.log1p(np.exp(-gate_scale * rng.standard_normal((B, T, H, dk)) + 1.0))
    elif variant == "gdn":
        loga = -np.log1p(np.exp(-gate_scale * rng.standard_normal((B, T, H)) + 1.0))
    else:
        loga = None
    S0 = 0.3 * rng.standard_normal((B, H, dk, dv)) if s0 else None
    return dict(q=q, k=k, v=v, loga=loga, beta=beta, S0=S0)


def channel_decay(loga, variant, dk):
    """alpha per (b,t,h,channel) as an array of shape [B,T,H,dk]."""
    if variant == "deltanet":
        return None
    a = np.exp(loga)
    if variant == "gdn":
        a = np.repeat(a[..., None], dk, axis=-1)
    return a


def close(a, b, tol, what):
    err = np.max(np.abs(np.asarray(a) - np.asarray(b))) if np.size(a) else 0.0
    scale = max(1.0, float(np.max(np.abs(b))) if np.size(b) else 1.0)
    assert err <= tol * scale, f"{what}: max|diff|={err:.3e} > {tol:.1e}*{scale:.3g}"


# --------------------------------------------------------------------------------------------
def pin_golden_hand_examples(lib):
    with open(GOLDEN) as f:
        g = json.load(f)
    c = g["common"]
    q = np.array(c["q"])[None, :, None, :]
    k = np.array(c["k"])[None, :, None, :]
    v = np.array(c["v"])[None, :, None, :]
    beta = np.array(c["beta"])[None, :, None]
    S0 = np.array(c["S0"])[None, None]
    for var, case in g["cases"].items():
        if case["alpha"] is None:
            loga = None
        else:
            a = np.array(case["alpha"])
            loga = np.log(a)[None, :, None, :] if a.ndim == 2 else np.log(a)[None, :, None]
        r = oracle.fwd(q, k, v, loga, beta, S0, variant=var, lib=lib)
        close(r["u"][0, :, 0], np.array(case["u"]), 1e-12, f"golden {var} u")
        close(r["o"][0, :, 0], np.array(case["o"]), 1e-12, f"golden {var} o")
        close(r["S_T"][0, 0], np.array(case["S_T"]), 1e-12, f"golden {var} S_T")
        rc = oracle.chunked_fwd(q, k, v, loga, beta, S0, variant=var, chunk=2, lib=lib)
        for key in ("u", "o"):
            close(rc[key][0, :, 0], np.array(case[key]), 1e-12, f"golden chunked {var} {key}")
        close(rc["S_T"][0, 0], np.array(case["S_T"]), 1e-12, f"golden chunked {var} S_T")


def pin_recall_orthonormal_keys(lib):
    """DeltaNet, alpha=1, beta=1, orthonormal keys: stored values are recalled exactly."""
    rng = np.random.default_rng(11)
    dk, dv, T = 8, 5, 8
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Qm.T[None, :, None, :].copy()  # rows are orthonormal keys
    v = rng.standard_normal((1, T, 1, dv))
    beta = np.ones((1, T, 1))
    for S0 in (None, rng.standard_normal((1, 1, dk, dv))):
        r = oracle.fwd(k, k, v, None, beta, S0, variant="deltanet", lib=lib)
        ST = r["S_T"][0, 0]
        close(ST.T @ k[0, :, 0].T, v[0, :, 0].T, 1e-12, "recall S_T^T k_i = v_i")
        pred0 = 0 if S0 is None else (S0[0, 0].T @ k[0, :, 0].T).T
        close(r["u"][0, :, 0], v[0, :, 0] - pred0, 1e-12, "u_t = v_t - S0^T k_t")
        # o_t = S_t^T q_t with q_t = k_t returns v_t
        close(r["o"][0, :, 0], v[0, :, 0], 1e-12, "o_t = v_t")


def pin_repeated_key_overwrites(lib):
    rng = np.random.default_rng(12)
    dk, dv = 6, 4
    kk = rng.standard_normal(dk)
    kk /= np.linalg.norm(kk)
    k = np.stack([kk, kk])[None, :, None, :]
    v = rng.standard_normal((1, 2, 1, dv))
    q = k.copy()
    r = oracle.fwd(q, k, v, None, np.ones((1, 2, 1)), None, variant="deltanet", lib=lib)
    close(r["u"][0, 1, 0], v[0, 1, 0] - v[0, 0, 0], 1e-12, "second write = v2 - v1")
    close(r["S_T"][0, 0].T @ kk, v[0, 1, 0], 1e-12, "key now recalls v2")


def pin_unit_key_beta_one_stores_value(lib):
    """Every variant: with beta=1 and |k_t|=1, S_t^T k_t = v_t, so q = k gives o_t = v_t."""
    rng = np.random.default_rng(13)
    for var in VARS:
        x = rand_inputs(rng, 2, 23, 3, 7, 5, var)
        x["beta"] = np.ones_like(x["beta"])
        r = oracle.fwd(x["k"], x["k"], x["v"], x["loga"], x["beta"], x["S0"], variant=var, lib=lib)
        close(r["o"], x["v"], 1e-11, f"{var}: o_t = v_t")


def pin_kda_uniform_equals_gdn(lib):
    rng = np.random.default_rng(14)
    x = rand_inputs(rng, 2, 19, 2, 6, 5, "gdn")
    lk = np.repeat(x["loga"][..., None], 6, axis=-1)
    a = oracle.fwd(x["q"], x["k"], x["v"], x["loga"], x["beta"], x["S0"], variant="gdn", lib=lib)
    b = oracle.fwd(x["q"], x["k"], x["v"], lk, x["beta"], x["S0"], variant="kda", lib=lib)
    for key in a:
        close(b[key], a[key], 1e-13, f"kda(uniform) == gdn {key}")
    # gradient consistency: the scalar gate's gradient is the channel sum of KDA's
    dO = rng.standard_normal(x["v"].shape)
    ga = oracle.bwd(**x, dO=dO, variant="gdn", lib=lib)
    gb = oracle.bwd(x["q"], x["k"], x["v"], lk, x["beta"], x["S0"], dO=dO, variant="kda", lib=lib)
    close(gb["dloga"].sum(-1), ga["dloga"], 1e-12, "sum_c dloga_kda == dloga_gdn")
    for key in ("dq", "dk", "dv", "dbeta", "dS0"):
        close(gb[key], ga[key], 1e-12, f"kda(uniform) grad == gdn grad {key}")


def pin_zero_gate_is_deltanet(lib):
    rng = np.random.default_rng(15)
    x = rand_inputs(rng, 1, 17, 2, 5, 4, "gdn")
    a = oracle.fwd(x["q"], x["k"], x["v"], np.zeros_like(x["loga"]), x["beta"], x["S0"], variant="gdn", lib=lib)
    b = oracle.fwd(x["q"], x["k"], x["v"], None, x["beta"], x["S0"], variant="deltanet", lib=lib)
    c = oracle.fwd(x["q"], x["k"], x["v"], x["loga"], x["beta"], x["S0"], variant="deltanet", lib=lib)
    for key in a:
        close(b[key], a[key], 1e-13, f"gdn(loga=0) == deltanet {key}")
        close(c[key], b[key], 0.0, f"deltanet ignores loga {key}")


def pin_beta_zero_is_pure_decay(lib):
    rng = np.random.default_rng(16)
    for var in ("gdn", "kda"):
        B, T, H, dk, dv = 1, 9, 2, 5, 3
        x = rand_inputs(rng, B, T, H, dk, dv, var)
        x["beta"] = np.zeros_like(x["beta"])
        r = oracle.fwd(**x, variant=var, lib=lib)
        a = channel_decay(x["loga"], var, dk)
        G = np.cumprod(a, axis=1)  # Gamma_{1:t} per channel
        for h in range(H):
            for t in range(T):
                St = G[0, t, h][:, None] * x["S0"][0, h]
                close(r["o"][0, t, h], St.T @ x["q"][0, t, h], 1e-13, f"{var} decay o")
            close(r["S_T"][0, h], G[0, T - 1, h][:, None] * x["S0"][0, h], 1e-13, f"{var} decay S_T")
        close(r["u"], np.zeros_like(r["u"]), 0.0, f"{var} decay u == 0")
        r0 = oracle.fwd(x["q"], x["k"], x["v"], x["loga"], x["beta"], None, variant=var, lib=lib)
        close(r0["o"], np.zeros_like(r0["o"]), 0.0, f"{var} zero state stays zero")


def pin_matrix_product_form(lib):
    """Step the section-2.1 equation literally with dense dk x dk matrices."""
    rng = np.random.default_rng(17)
    for var in VARS:
        B, T, H, dk, dv = 1, 8, 2, 4, 3
        x = rand_inputs(rng, B, T, H, dk, dv, var, unit_keys=False)
        r = oracle.fwd(**x, variant=var, lib=lib)
        a = channel_decay(x["loga"], var, dk)
        for h in range(H):
            S = x["S0"][0, h].copy()
            for t in range(T):
                kt = x["k"][0, t, h][:, None]
                bt = x["beta"][0, t, h]
                D = np.eye(dk) if a is None else np.diag(a[0, t, h])
                u_ref = bt * (x["v"][0, t, h] - (D @ S).T @ kt[:, 0])
                S = (np.eye(dk) - bt * kt @ kt.T) @ D @ S + bt * kt @ x["v"][0, t, h][None, :]
                close(r["u"][0, t, h], u_ref, 1e-12, f"{var} matrix-form u t={t}")
                close(r["o"][0, t, h], S.T @ x["q"][0, t, h], 1e-12, f"{var} matrix-form o t={t}")
            close(r["S_T"][0, h], S, 1e-12, f"{var} matrix-form S_T")


def pin_chunked_matches_recurrence(lib):
    rng = np.random.default_rng(18)
    for var in VARS:
        x = rand_inputs(rng, 2, 37, 2, 6, 5, var, gate_scale=2.0)
        ref = oracle.fwd(**x, variant=var, lib=lib)
        for C in (1, 4, 8, 16, 64):
            r = oracle.chunked_fwd(**x, variant=var, chunk=C, lib=lib)
            for key in ref:
                close(r[key], ref[key], 1e-11, f"{var} chunk={C} {key}")


def pin_linear_in_state_and_values(lib):
    rng = np.random.default_rng(19)
    for var in VARS:
        x = rand_inputs(rng, 1, 13, 2, 5, 4, var)
        y = dict(x, v=rng.standard_normal(x["v"].shape), S0=rng.standard_normal(x["S0"].shape))
        z = dict(x, v=2.0 * x["v"] - 3.0 * y["v"], S0=2.0 * x["S0"] - 3.0 * y["S0"])
        rx, ry, rz = (oracle.fwd(**w, variant=var, lib=lib) for w in (x, y, z))
        for key in rx:
            close(rz[key], 2.0 * rx[key] - 3.0 * ry[key], 1e-12, f"{var} linearity {key}")


def pin_split_sequence(lib):
    rng = np.random.default_rng(20)
    for var in VARS:
        x = rand_inputs(rng, 2, 30, 2, 5, 4, var)
        full = oracle.fwd(**x, variant=var, lib=lib)
        for t1 in (1, 11, 29):
            first = {key: (val[:, :t1] if key not in ("S0",) and val is not None else val) for key, val in x.items()}
            second = {key: (val[:, t1:] if key not in ("S0",) and val is not None else val) for key, val in x.items()}
            a = oracle.fwd(**first, variant=var, lib=lib)
            second["S0"] = a["S_T"]
            b = oracle.fwd(**second, variant=var, lib=lib)
            close(np.concatenate([a["o"], b["o"]], 1), full["o"], 1e-12, f"{var} split o")
            close(np.concatenate([a["u"], b["u"]], 1), full["u"], 1e-12, f"{var} split u")
            close(b["S_T"], full["S_T"], 1e-12, f"{var} split S_T")


def pin_state_from_write_values(lib):
    """S_T = Gamma_{1:T} S0 + sum_t Gamma_{t+1:T} k_t u_t^T."""
    rng = np.random.default_rng(21)
    for var in VARS:
        B, T, H, dk, dv = 1, 21, 2, 6, 4
        x = rand_inputs(rng, B, T, H, dk, dv, var)
        r = oracle.fwd(**x, variant=var, lib=lib)
        a = channel_decay(x["loga"], var, dk)
        if a is None:
            a = np.ones((B, T, H, dk))
        for h in range(H):
            S = np.prod(a[0, :, h], axis=0)[:, None] * x["S0"][0, h]
            for t in range(T):
                tail = np.prod(a[0, t + 1:, h], axis=0) if t + 1 < T else np.ones(dk)
                S = S + (tail * x["k"][0, t, h])[:, None] * r["u"][0, t, h][None, :]
            close(r["S_T"][0, h], S, 1e-12, f"{var} reconstruction")


def pin_t1_closed_forms(lib):
    """One token from a zero state: u = beta v, S = beta k v^T, o = beta (k.q) v, and its gradients."""
    rng = np.random.default_rng(22)
    dk, dv = 5, 3
    q, k = rng.standard_normal((1, 1, 1, dk)), rng.standard_normal((1, 1, 1, dk))
    v = rng.standard_normal((1, 1, 1, dv))
    b = np.array([[[0.7]]])
    r = oracle.fwd(q, k, v, None, b, None, variant="deltanet", lib=lib)
    kq = float(k.ravel() @ q.ravel())
    close(r["u"].ravel(), 0.7 * v.ravel(), 1e-14, "T1 u")
    close(r["o"].ravel(), 0.7 * kq * v.ravel(), 1e-14, "T1 o")
    close(r["S_T"][0, 0], 0.7 * np.outer(k.ravel(), v.ravel()), 1e-14, "T1 S")
    dO, du, dS = rng.standard_normal(dv), rng.standard_normal(dv), rng.standard_normal((dk, dv))
    g = oracle.bwd(q, k, v, None, b, None, dO[None, None, None], du[None, None, None], dS[None, None],
                   variant="deltanet", lib=lib)
    kk, vv, qq = k.ravel(), v.ravel(), q.ravel()
    close(g["dq"].ravel(), 0.7 * (vv @ dO) * kk, 1e-13, "T1 dq")
    close(g["dk"].ravel(), 0.7 * (vv @ dO) * qq + 0.7 * dS @ vv, 1e-13, "T1 dk")
    close(g["dv"].ravel(), 0.7 * kq * dO + 0.7 * du + 0.7 * dS.T @ kk, 1e-13, "T1 dv")
    close(g["dbeta"].ravel(), [kq * (vv @ dO) + vv @ du + kk @ dS @ vv], 1e-13, "T1 dbeta")
    close(g["dS0"][0, 0], np.zeros((dk, dv)) + (np.eye(dk) - 0.7 * np.outer(kk, kk)) @ (
        np.outer(qq, dO) + dS) - 0.7 * np.outer(kk, du), 1e-13, "T1 dS0")


def _loss(r, dO, du, dS):
    L = float(np.sum(r["o"] * dO)) + float(np.sum(r["S_T"] * dS))
    if du is not None:
        L += float(np.sum(r["u"] * du))
    return L


def pin_backward_finite_differences(lib, T=9, dk=4, dv=3, ndir=3):
    """Central differences of L = <dO,o> + <du,u> + <dS_T,S_T> along random directions."""
    rng = np.random.default_rng(23)
    for var in VARS:
        x = rand_inputs(rng, 1, T, 2, dk, dv, var, unit_keys=False)
        dO = rng.standard_normal(x["v"].shape)
        du = rng.standard_normal(x["v"].shape)
        dS = rng.standard_normal(x["S0"].shape)
        g = oracle.bwd(**x, dO=dO, du=du, dS_T=dS, variant=var, lib=lib)
        names = [("q", "dq"), ("k", "dk"), ("v", "dv"), ("beta", "dbeta"), ("S0", "dS0")]
        if var != "deltanet":
            names.append(("loga", "dloga"))
        h = 1e-6
        for name, gname in names:
            for _ in range(ndir):
                d = rng.standard_normal(x[name].shape)
                xp = dict(x)
                xm = dict(x)
                xp[name] = x[name] + h * d
                xm[name] = x[name] - h * d
                fd = (_loss(oracle.fwd(**xp, variant=var, lib=lib), dO, du, dS)
                      - _loss(oracle.fwd(**xm, variant=var, lib=lib), dO, du, dS)) / (2 * h)
                an = float(np.sum(g[gname] * d))
                assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), f"{var} FD {name}: fd={fd:.9g} analytic={an:.9g}"
        if var == "deltanet":
            close(g["dloga"], np.zeros_like(g["dloga"]), 0.0, "deltanet has no gate gradient")


def pin_adjoint_identity(lib):
    """(S0, V) -> (o, u, S_T) is linear; its adjoint is the backward: <J x, w> = <x, J^T w>."""
    rng = np.random.default_rng(24)
    for var in VARS:
        x = rand_inputs(rng, 2, 15, 2, 5, 4, var)
        wO, wu, wS = (rng.standard_normal(s) for s in (x["v"].shape, x["v"].shape, x["S0"].shape))
        r = oracle.fwd(**x, variant=var, lib=lib)
        g = oracle.bwd(**x, dO=wO, du=wu, dS_T=wS, variant=var, lib=lib)
        lhs = np.sum(r["o"] * wO) + np.sum(r["u"] * wu) + np.sum(r["S_T"] * wS)
        rhs = np.sum(x["S0"] * g["dS0"]) + np.sum(x["v"] * g["dv"])
        assert abs(lhs - rhs) <= 1e-11 * max(1.0, abs(lhs)), f"{var} adjoint: {lhs} vs {rhs}"


ALL_PINS = [
    pin_golden_hand_examples,
    pin_recall_orthonormal_keys,
    pin_repeated_key_overwrites,
    pin_unit_key_beta_one_stores_value,
    pin_kda_uniform_equals_gdn,
    pin_zero_gate_is_deltanet,
    pin_beta_zero_is_pure_decay,
    pin_matrix_product_form,
    pin_chunked_matches_recurrence,
    pin_linear_in_state_and_values,
    pin_split_sequence,
    pin_state_from_write_values,
    pin_t1_closed_forms,
    pin_backward_finite_differences,
    pin_adjoint_identity,
]
