"""Depthwise causal short convolution over the token axis, in plain fp64 numpy.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: the independent checker for the CUDA
library's short-convolution kernels (gated_delta_rule_107_b200/csrc/shortconv.cu).  It shares no
code with the library, and the product path never calls it; only tests/ and bench.py's CPU legs
use it.

"线性注意力架构演进与Kimi Delta Attention创新实践", section 4.2: a depthwise convolution of kernel
size 4 on the q/k/v path picks up local (n-gram) patterns.  Reading taken (the page gives the
kernel size and that it is depthwise, nothing else): every channel c of a token-major stream
x [B, T, D] is filtered causally with its own four taps w[c, 0..3], the last tap on the
current token,
    y[b, t, c] = sum_{j=0..3} w[c, j] * x[b, t - 3 + j, c],
with x at t < 0 taken from a three-token cache x_prev [B, 3, D] (row 3 + t) or zero when there
is none; no bias, no activation (the page names neither).  The returned cache is the last three
tokens of [x_prev ; x], what a later call on the continuation of the stream takes as x_prev.

Backward of L = sum(dy * y) (dy past the last token is zero):
    dx[b, s, c] = sum_j w[c, j] dy[b, s + 3 - j, c]      for s = -3 .. T-1 (s < 0: dx_prev)
    dw[c, j]    = sum_{b, t} dy[b, t, c] x[b, t - 3 + j, c]
"""
from __future__ import annotations

import numpy as np

K = 4  # taps


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def _padded(x, x_prev):
    """[x_prev ; x] along the token axis: row t + 3 holds token t."""
    B, _, D = x.shape
    prev = np.zeros((B, K - 1, D)) if x_prev is None else _f64(x_prev)
    return np.concatenate([prev, x], axis=1)


def shortconv_fwd(x, w, x_prev=None):
    """Returns (y [B, T, D], cache [B, 3, D])."""
    x, w = _f64(x), _f64(w)
    T = x.shape[1]
    xp = _padded(x, x_prev)
    y = np.zeros(x.shape)
    for j in range(K):  # token t - 3 + j sits at row t + j of xp
        y += w[:, j] * xp[:, j:j + T]
    return y, xp[:, T:].copy()


def shortconv_bwd(x, w, dy, x_prev=None):
    """Returns dict(dx [B, T, D], dw [D, 4], dx_prev [B, 3, D])."""
    x, w, dy = _f64(x), _f64(w), _f64(dy)
    B, T, D = x.shape
    xp = _padded(x, x_prev)
    dxp = np.zeros((B, T + K - 1, D))
    dw = np.zeros((D, K))
    for j in range(K):
        dxp[:, j:j + T] += w[:, j] * dy
        dw[:, j] = np.sum(dy * xp[:, j:j + T], axis=(0, 1))
    return {"dx": dxp[:, K - 1:], "dw": dw, "dx_prev": dxp[:, :K - 1]}
