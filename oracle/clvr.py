"""Cross-layer value routing (CLVR): a lower layer's write values added, through a projection,
to a higher layer's hidden stream, in plain fp64 numpy.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: the independent checker for the CUDA
library's routing entry points (gated_delta_rule_107_b200/csrc/clvr.cu).  It shares no code
with the library, and the product path never calls it; only tests/ and bench.py's CPU legs use
it.

ETH news page on the architecture study, section 七 (and the explainer's CLVR section): the
signal routed upward is the write value u_t = beta_t (v_t - S'_t^T k_t) (not the write error),
it enters the residual stream shared by all layers, and the projection matrix starts at zero,
so that at initialisation the network is exactly the one without routing.  With U the write
values as a [B*T, H*dv] matrix, W the projection [H*dv, D] and h the receiving hidden stream
[B*T, D]:
    h_out = h + U W
Backward of L = sum(dh_out * h_out): dU = dh_out W^T, dW = U^T dh_out, dh = dh_out.
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def clvr_fwd(u, W, h=None):
    """h_out [M, N] for u [M, K] (or [B, T, H, dv] with K = H dv), W [K, N], h [M, N] or None (zero)."""
    W = _f64(W)
    U = _f64(u).reshape(-1, W.shape[0])
    out = U @ W
    if h is not None:
        out = out + _f64(h).reshape(out.shape)
    return out


def clvr_bwd(u, W, dh_out):
    """Returns dict(du [M, K], dW [K, N]); the gradient of h is dh_out itself."""
    W = _f64(W)
    U = _f64(u).reshape(-1, W.shape[0])
    dH = _f64(dh_out).reshape(U.shape[0], W.shape[1])
    return {"du": dH @ W.T, "dW": U.T @ dH}
