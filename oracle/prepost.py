"""Operations just before and just after the delta-rule core, in plain fp64 numpy.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: the independent checker for the
CUDA library's pre/post kernels (gated_delta_rule_107_b200/csrc/prepost.cu).  It shares no
code with the library, and the product path never calls it; only tests/ and bench.py's
CPU legs use it.  Every function is the plain definition, written out step by step.

Pre-operations ("线性注意力架构演进与Kimi Delta Attention创新实践", section 7.1 -- q and k
are L2-normalised after their projections, the forget gate carries a bias of -3 so that
it starts near sigmoid(-3) ~ 0.05, and decay is handled in log space; section 2.1 --
beta_t in (0, 1)), per (token, head) row:
    q_hat = q / sqrt(sum(q^2) + eps),   k_hat = k / sqrt(sum(k^2) + eps)
    beta  = sigmoid(b)                                  (raw write-strength logit b)
    log alpha = -softplus(a) = log(1 - sigmoid(a))      (raw forget logit a; alpha is
                                                         the retained fraction)
Post-operation (same page, section 4.1: the output gate Sigmoid(W x) applied to
RMSNorm of the attention output), per (token, head) row of dv channels:
    n = o / sqrt(mean(o^2) + eps),   y = n * w * sigmoid(g)
with a per-channel weight w and the gate logits g given by the caller.

eps = 1e-6 in both (the method's description gives no value).  The backward functions return the gradients of
L = sum(dy * y) (post) or of L = <dq_hat, q_hat> + <dk_hat, k_hat> + <dbeta, beta> +
<dloga, log alpha> (pre) with respect to every input.
"""
from __future__ import annotations

import numpy as np

EPS = 1e-6


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def _sigmoid(x):
    # split by sign so that exp never overflows
    out = np.empty_like(x)
    pos = x >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-x[pos]))
    ex = np.exp(x[~pos])
    out[~pos] = ex / (1.0 + ex)
    return out


def _softplus(x):
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def l2norm_fwd(x):
    """x / sqrt(sum(x^2) + eps) over the last axis."""
    x = _f64(x)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + EPS)


def l2norm_bwd(x, dy):
    """Gradient of <dy, l2norm(x)> with respect to x."""
    x, dy = _f64(x), _f64(dy)
    r = np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + EPS)
    y = x / r
    return (dy - y * np.sum(y * dy, axis=-1, keepdims=True)) / r


def preop_fwd(q, k, b, a=None):
    """Returns dict(q, k, beta, loga); loga is None when there is no gate (DeltaNet)."""
    b = _f64(b)
    a = _f64(a)
    return {"q": l2norm_fwd(q), "k": l2norm_fwd(k), "beta": _sigmoid(b),
            "loga": None if a is None else -_softplus(a)}


def preop_bwd(q, k, b, a, dq, dk, dbeta, dloga):
    """Gradients with respect to the raw q, k, b, a (da is None when a is None)."""
    b = _f64(b)
    beta = _sigmoid(b)
    out = {"dq": l2norm_bwd(q, dq), "dk": l2norm_bwd(k, dk), "db": _f64(dbeta) * beta * (1.0 - beta), "da": None}
    if a is not None:
        out["da"] = -_f64(dloga) * _sigmoid(_f64(a))
    return out


def postop_fwd(o, g, w=None):
    """y = rmsnorm(o) * w * sigmoid(g) over the last axis (w = 1 when None)."""
    o, g = _f64(o), _f64(g)
    w = np.ones(o.shape[-1]) if w is None else _f64(w)
    n = o / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + EPS)
    return n * w * _sigmoid(g)


def postop_bwd(o, g, w, dy):
    """Returns dict(do, dg, dw) for L = sum(dy * y); dw sums over every row."""
    o, g, dy = _f64(o), _f64(g), _f64(dy)
    d = o.shape[-1]
    w = np.ones(d) if w is None else _f64(w)
    r = 1.0 / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + EPS)
    n = o * r
    s = _sigmoid(g)
    dz = dy * s                     # d(n * w)
    dg = dy * n * w * s * (1.0 - s)
    dw = np.sum((dz * n).reshape(-1, d), axis=0)
    dn = dz * w
    do = r * (dn - n * np.mean(dn * n, axis=-1, keepdims=True))
    return {"do": do, "dg": dg, "dw": dw}
