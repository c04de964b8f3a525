"""ctypes binding of libdeltarule.so (the C ABI in include/delta_rule.h).

Argument marshalling only: every step of the computation runs in the library's
CUDA kernels.  PyTorch supplies device memory and the current stream.  There is
no fallback: if the shared library is missing or a call fails, an exception is
raised.

Low level: ``workspace_size``, ``saved_size``, ``fwd_raw``, ``bwd_raw``,
``fwd_save_raw``, ``bwd_saved_raw``, ``strerror``, ``sync_status`` mirror the C
entry points one to one (integer pointers).
High level: ``delta_rule_fwd`` / ``delta_rule_bwd`` take torch CUDA tensors,
allocate outputs and the workspace with torch, and call the C ABI on the
current stream; ``delta_rule_fwd_save`` / ``delta_rule_bwd_saved`` are the
training pair (the forward keeps what the backward would recompute in a saved
buffer); ``delta_rule_decode`` is the recurrent form for the few tokens of a
decoding step (state in, state out, optionally in place); ``delta_rule_preop`` /
``delta_rule_postop`` and their ``_bwd`` are the single-pass operations just
before and after the core (L2-normalised q, k, logistic gates; sigmoid-gated
RMSNorm of the output).  ``delta_rule_fwd_host``
is the forward for host tensors (copies in, computes, copies out).

The ``for_bwd`` argument of ``workspace_size`` and ``launches`` names the call:
0 forward, 1 backward, 2 saving forward, 3 backward from saved activations.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

DR_DELTANET, DR_GATED, DR_KDA = 0, 1, 2
DR_F32, DR_BF16 = 0, 1
DR_OK, DR_ERR_ARG, DR_ERR_UNSUPPORTED, DR_ERR_ALIGN, DR_ERR_WORKSPACE, DR_ERR_CUDA, DR_ERR_TIMEOUT = 0, -1, -2, -3, -4, -5, -6
VARIANTS = {"deltanet": DR_DELTANET, "gdn": DR_GATED, "gated": DR_GATED, "kda": DR_KDA}
DTYPES = {torch.float32: DR_F32, torch.bfloat16: DR_BF16}

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdeltarule.so")
EXPORTS = ("delta_rule_workspace_size", "delta_rule_fwd", "delta_rule_bwd", "delta_rule_strerror",
           "delta_rule_sync_status", "delta_rule_launches", "delta_rule_fwd_timed", "delta_rule_bwd_timed",
           "delta_rule_fwd_noalloc", "delta_rule_saved_size", "delta_rule_fwd_save", "delta_rule_bwd_saved",
           "delta_rule_fwd_save_timed", "delta_rule_bwd_saved_timed", "delta_rule_decode",
           "delta_rule_preop", "delta_rule_preop_bwd", "delta_rule_postop_workspace_size", "delta_rule_postop",
           "delta_rule_postop_bwd", "delta_rule_selftest_timeout", "delta_rule_shortconv_workspace_size",
           "delta_rule_shortconv", "delta_rule_shortconv_bwd", "delta_rule_clvr_workspace_size", "delta_rule_clvr",
           "delta_rule_clvr_bwd", "delta_rule_fwd_fused_workspace_size", "delta_rule_fwd_fused")

_lib = None


class DeltaRuleError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {strerror(code)} ({code})")
        self.code = code


def load(path: str | None = None):
    """Load libdeltarule.so (built by gated_delta_rule_107_b200.build); raises if it is absent."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise ImportError(f"{p} not found: build it with `python -m gated_delta_rule_107_b200.build` "
                          "(the CUDA library is required; there is no fallback)")
    lib = ctypes.CDLL(p)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.delta_rule_workspace_size.argtypes = [i] * 9
    lib.delta_rule_workspace_size.restype = sz
    lib.delta_rule_fwd.argtypes = [vp] * 9 + [i] * 8 + [vp, sz, vp]
    lib.delta_rule_fwd.restype = i
    lib.delta_rule_bwd.argtypes = [vp] * 15 + [i] * 8 + [vp, sz, vp]
    lib.delta_rule_bwd.restype = i
    lib.delta_rule_strerror.argtypes = [i]
    lib.delta_rule_strerror.restype = ctypes.c_char_p
    lib.delta_rule_sync_status.argtypes = [vp]
    lib.delta_rule_sync_status.restype = i
    lib.delta_rule_launches.argtypes = [i] * 9 + [ctypes.POINTER(ctypes.c_char_p), i]
    lib.delta_rule_launches.restype = i
    lib.delta_rule_plain_launches.argtypes = [i] * 9
    lib.delta_rule_plain_launches.restype = i
    lib.delta_rule_fwd_timed.argtypes = [vp] * 9 + [i] * 8 + [vp, sz, vp, ctypes.POINTER(vp), i]
    lib.delta_rule_fwd_timed.restype = i
    lib.delta_rule_bwd_timed.argtypes = [vp] * 15 + [i] * 8 + [vp, sz, vp, ctypes.POINTER(vp), i]
    lib.delta_rule_bwd_timed.restype = i
    lib.delta_rule_fwd_noalloc.argtypes = [vp] * 9 + [i] * 8 + [vp]
    lib.delta_rule_fwd_noalloc.restype = i
    lib.delta_rule_saved_size.argtypes = [i] * 8
    lib.delta_rule_saved_size.restype = sz
    lib.delta_rule_fwd_save.argtypes = [vp] * 9 + [i] * 8 + [vp, sz, vp, sz, vp]
    lib.delta_rule_fwd_save.restype = i
    lib.delta_rule_bwd_saved.argtypes = [vp] * 15 + [i] * 8 + [vp, sz, vp, sz, vp]
    lib.delta_rule_bwd_saved.restype = i
    lib.delta_rule_preop.argtypes = [vp] * 8 + [i] * 6 + [vp]
    lib.delta_rule_preop.restype = i
    lib.delta_rule_preop_bwd.argtypes = [vp] * 12 + [i] * 6 + [vp]
    lib.delta_rule_preop_bwd.restype = i
    lib.delta_rule_postop_workspace_size.argtypes = [i]
    lib.delta_rule_postop_workspace_size.restype = sz
    lib.delta_rule_postop.argtypes = [vp] * 4 + [i] * 5 + [vp]
    lib.delta_rule_postop.restype = i
    lib.delta_rule_postop_bwd.argtypes = [vp] * 7 + [i] * 5 + [vp, sz, vp]
    lib.delta_rule_postop_bwd.restype = i
    lib.delta_rule_shortconv_workspace_size.argtypes = [i] * 3
    lib.delta_rule_shortconv_workspace_size.restype = sz
    lib.delta_rule_shortconv.argtypes = [vp] * 5 + [i] * 4 + [vp]
    lib.delta_rule_shortconv.restype = i
    lib.delta_rule_shortconv_bwd.argtypes = [vp] * 7 + [i] * 4 + [vp, sz, vp]
    lib.delta_rule_shortconv_bwd.restype = i
    lib.delta_rule_clvr_workspace_size.argtypes = []
    lib.delta_rule_clvr_workspace_size.restype = sz
    lib.delta_rule_clvr.argtypes = [vp] * 4 + [i] * 4 + [vp, sz, vp]
    lib.delta_rule_clvr.restype = i
    lib.delta_rule_clvr_bwd.argtypes = [vp] * 5 + [i] * 4 + [vp, sz, vp]
    lib.delta_rule_clvr_bwd.restype = i
    lib.delta_rule_selftest_timeout.argtypes = [ctypes.c_uint, vp]
    lib.delta_rule_selftest_timeout.restype = i
    lib.delta_rule_decode.argtypes = [vp] * 9 + [i] * 7 + [vp]
    lib.delta_rule_decode.restype = i
    lib.delta_rule_fwd_save_timed.argtypes = [vp] * 9 + [i] * 8 + [vp, sz, vp, sz, vp, ctypes.POINTER(vp), i]
    lib.delta_rule_fwd_save_timed.restype = i
    lib.delta_rule_bwd_saved_timed.argtypes = [vp] * 15 + [i] * 8 + [vp, sz, vp, sz, vp, ctypes.POINTER(vp), i]
    lib.delta_rule_bwd_saved_timed.restype = i
    lib.delta_rule_fwd_fused_workspace_size.argtypes = [i] * 8
    lib.delta_rule_fwd_fused_workspace_size.restype = sz
    lib.delta_rule_fwd_fused.argtypes = [vp] * 12 + [i] * 8 + [vp, sz, vp]
    lib.delta_rule_fwd_fused.restype = i
    if path is None:
        _lib = lib
    return lib


def strerror(code: int) -> str:
    return load().delta_rule_strerror(int(code)).decode()


def workspace_size(B, T, H, dk, dv, variant, chunk, dtype, for_bwd) -> int:
    n = load().delta_rule_workspace_size(B, T, H, dk, dv, variant, chunk, dtype, int(for_bwd))
    if n == ctypes.c_size_t(-1).value:
        raise DeltaRuleError(DR_ERR_ARG, "delta_rule_workspace_size")
    return n


def saved_size(B, T, H, dk, dv, variant, chunk, dtype) -> int:
    """Bytes of the saved-activation buffer (0: this configuration has no saved form)."""
    n = load().delta_rule_saved_size(B, T, H, dk, dv, variant, chunk, dtype)
    if n == ctypes.c_size_t(-1).value:
        raise DeltaRuleError(DR_ERR_ARG, "delta_rule_saved_size")
    return n


def plain_launches(B, T, H, dk, dv, variant, chunk, dtype, for_bwd) -> int:
    """How many kernels the plain entry point launches (more than ``launches`` when it runs in segments)."""
    n = load().delta_rule_plain_launches(B, T, H, dk, dv, variant, chunk, dtype, int(for_bwd))
    if n < 0:
        raise DeltaRuleError(n, "delta_rule_plain_launches")
    return n


def launches(B, T, H, dk, dv, variant, chunk, dtype, for_bwd) -> list[str]:
    """Names of the kernels one call launches, in launch order."""
    names = (ctypes.c_char_p * 16)()
    n = load().delta_rule_launches(B, T, H, dk, dv, variant, chunk, dtype, int(for_bwd), names, 16)
    if n < 0:
        raise DeltaRuleError(n, "delta_rule_launches")
    return [names[i].decode() for i in range(n)]


def event_array(events):
    """ctypes array of the raw cudaEvent_t handles of torch.cuda.Event objects."""
    arr = (ctypes.c_void_p * len(events))()
    for i, e in enumerate(events):
        arr[i] = e.cuda_event
    return arr


def fwd_raw(*args) -> int:
    return load().delta_rule_fwd(*args)


def bwd_raw(*args) -> int:
    return load().delta_rule_bwd(*args)


def fwd_noalloc_raw(*args) -> int:
    """delta_rule_fwd_noalloc: the forward with the library's built-in scratch (no workspace argument)."""
    return load().delta_rule_fwd_noalloc(*args)


def fwd_timed_raw(*args) -> int:
    return load().delta_rule_fwd_timed(*args)


def bwd_timed_raw(*args) -> int:
    return load().delta_rule_bwd_timed(*args)


def fwd_save_raw(*args) -> int:
    return load().delta_rule_fwd_save(*args)


def bwd_saved_raw(*args) -> int:
    return load().delta_rule_bwd_saved(*args)


def fwd_save_timed_raw(*args) -> int:
    return load().delta_rule_fwd_save_timed(*args)


def bwd_saved_timed_raw(*args) -> int:
    return load().delta_rule_bwd_saved_timed(*args)


def sync_status(stream=None) -> int:
    s = torch.cuda.current_stream().cuda_stream if stream is None else stream
    return load().delta_rule_sync_status(s)


# ------------------------------------------------------------------------------------------------
def _p(t):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("delta_rule tensors must be contiguous (the C ABI takes dense [B,T,H,d] / [B,H,dk,dv])")
    return t.data_ptr()


def _variant(v) -> int:
    return VARIANTS[v] if isinstance(v, str) else int(v)


def _check(code, what):
    if code != DR_OK:
        raise DeltaRuleError(code, what)


def _workspace(nbytes: int, device) -> torch.Tensor | None:
    if nbytes == 0:
        return None
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def delta_rule_fwd(q, k, v, alpha, beta, S0=None, variant="gdn", chunk=64, want_u=True, want_state=True,
                   workspace: torch.Tensor | None = None, out=None, u=None, S_T=None):
    """Forward on CUDA tensors.  Returns (o, u or None, S_T or None).

    q, k: [B,T,H,dk]; v: [B,T,H,dv]; alpha: log gate [B,T,H] (gdn) / [B,T,H,dk] (kda) / None (deltanet);
    beta: [B,T,H]; S0: fp32 [B,H,dk,dv] or None.  All per-token tensors share one dtype (fp32 or bf16).
    """
    var = _variant(variant)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = DTYPES[q.dtype]
    dev = q.device
    out = torch.empty((B, T, H, dv), dtype=q.dtype, device=dev) if out is None else out
    if want_u and u is None:
        u = torch.empty((B, T, H, dv), dtype=q.dtype, device=dev)
    if want_state and S_T is None:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    need = workspace_size(B, T, H, dk, dv, var, chunk, dt, 0)
    if workspace is None or workspace.numel() < need:
        workspace = _workspace(need, dev)
    stream = torch.cuda.current_stream(dev).cuda_stream
    rc = fwd_raw(_p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(S0), _p(out), _p(u), _p(S_T),
                 B, T, H, dk, dv, var, chunk, dt, _p(workspace), need, stream)
    _check(rc, "delta_rule_fwd")
    return out, u, S_T


def selftest_timeout(limit_us: int, stream=None) -> int:
    """Runs the bounded-wait self-test (see include/delta_rule.h); returns the launch status."""
    return load().delta_rule_selftest_timeout(int(limit_us), stream)


def decode_raw(*args) -> int:
    return load().delta_rule_decode(*args)


def delta_rule_decode(q, k, v, alpha, beta, S=None, variant="gdn", want_u=True, inplace=False, out=None, u=None,
                      S_out=None):
    """Recurrent step(s) for decoding on CUDA tensors.  Returns (o, u or None, S_out).

    Shapes as delta_rule_fwd; S: fp32 [B,H,dk,dv] or None (zero state).  With inplace=True the
    state is updated in S itself (S_out is S)."""
    var = _variant(variant)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = DTYPES[q.dtype]
    dev = q.device
    out = torch.empty((B, T, H, dv), dtype=q.dtype, device=dev) if out is None else out
    if want_u and u is None:
        u = torch.empty((B, T, H, dv), dtype=q.dtype, device=dev)
    if inplace:
        if S is None:
            raise ValueError("inplace decoding needs a state tensor")
        S_out = S
    elif S_out is None:
        S_out = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev).cuda_stream
    rc = decode_raw(_p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(S), _p(S_out), _p(out), _p(u),
                    B, T, H, dk, dv, var, dt, stream)
    _check(rc, "delta_rule_decode")
    return out, u, S_out


def preop_raw(*args) -> int:
    return load().delta_rule_preop(*args)


def preop_bwd_raw(*args) -> int:
    return load().delta_rule_preop_bwd(*args)


def postop_raw(*args) -> int:
    return load().delta_rule_postop(*args)


def postop_bwd_raw(*args) -> int:
    return load().delta_rule_postop_bwd(*args)


def delta_rule_preop(q_raw, k_raw, beta_raw, gate_raw=None, variant="gdn"):
    """The core's inputs from raw projections: (q, k, beta, loga); loga is None for deltanet."""
    var = _variant(variant)
    B, T, H, dk = q_raw.shape
    q, k, beta = torch.empty_like(q_raw), torch.empty_like(k_raw), torch.empty_like(beta_raw)
    loga = torch.empty_like(gate_raw) if (var != DR_DELTANET and gate_raw is not None) else None
    rc = preop_raw(_p(q_raw), _p(k_raw), _p(beta_raw), _p(gate_raw), _p(q), _p(k), _p(beta), _p(loga), B, T, H, dk,
                   var, DTYPES[q_raw.dtype], torch.cuda.current_stream(q_raw.device).cuda_stream)
    _check(rc, "delta_rule_preop")
    return q, k, beta, loga


def delta_rule_preop_bwd(q_raw, k_raw, beta_raw, gate_raw, dq, dk, dbeta, dloga=None, variant="gdn"):
    """Gradients with respect to (q_raw, k_raw, beta_raw, gate_raw); the last is None for deltanet."""
    var = _variant(variant)
    B, T, H, dk_ = q_raw.shape
    gq, gk, gb = torch.empty_like(q_raw), torch.empty_like(k_raw), torch.empty_like(beta_raw)
    ga = torch.empty_like(gate_raw) if (var != DR_DELTANET and gate_raw is not None) else None
    rc = preop_bwd_raw(_p(q_raw), _p(k_raw), _p(beta_raw), _p(gate_raw), _p(dq), _p(dk), _p(dbeta), _p(dloga),
                       _p(gq), _p(gk), _p(gb), _p(ga), B, T, H, dk_, var, DTYPES[q_raw.dtype],
                       torch.cuda.current_stream(q_raw.device).cuda_stream)
    _check(rc, "delta_rule_preop_bwd")
    return gq, gk, gb, ga


def delta_rule_postop(o, gate, weight=None):
    """y = rmsnorm(o) * weight * sigmoid(gate) per (token, head) row."""
    B, T, H, dv = o.shape
    y = torch.empty_like(o)
    rc = postop_raw(_p(o), _p(gate), _p(weight), _p(y), B, T, H, dv, DTYPES[o.dtype],
                    torch.cuda.current_stream(o.device).cuda_stream)
    _check(rc, "delta_rule_postop")
    return y


def delta_rule_postop_bwd(o, gate, weight, dy, want_dweight=True):
    """Returns (do, dgate, dweight or None)."""
    B, T, H, dv = o.shape
    go, gg = torch.empty_like(o), torch.empty_like(gate)
    gw = torch.empty(dv, dtype=torch.float32, device=o.device) if want_dweight else None
    need = load().delta_rule_postop_workspace_size(dv)
    ws = _workspace(need, o.device)
    rc = postop_bwd_raw(_p(o), _p(gate), _p(weight), _p(dy), _p(go), _p(gg), _p(gw), B, T, H, dv, DTYPES[o.dtype],
                        _p(ws), need, torch.cuda.current_stream(o.device).cuda_stream)
    _check(rc, "delta_rule_postop_bwd")
    return go, gg, gw


def shortconv_raw(*args) -> int:
    return load().delta_rule_shortconv(*args)


def shortconv_bwd_raw(*args) -> int:
    return load().delta_rule_shortconv_bwd(*args)


def _stream_shape(x):
    """(B, T, D) of a [B, T, D] or [B, T, H, d] stream."""
    return x.shape[0], x.shape[1], math.prod(x.shape[2:])


def delta_rule_shortconv(x, weight, x_prev=None, want_cache=False):
    """Kernel-4 depthwise causal convolution along the tokens of x ([B, T, D] or [B, T, H, d]), taps
    weight [D, 4] fp32.  Returns y, or (y, cache) with cache [B, 3, D] when want_cache."""
    B, T, D = _stream_shape(x)
    y = torch.empty_like(x)
    cache = torch.empty((B, 3, D), dtype=x.dtype, device=x.device) if want_cache else None
    rc = shortconv_raw(_p(x), _p(weight), _p(x_prev), _p(y), _p(cache), B, T, D, DTYPES[x.dtype],
                       torch.cuda.current_stream(x.device).cuda_stream)
    _check(rc, "delta_rule_shortconv")
    return (y, cache) if want_cache else y


def delta_rule_shortconv_bwd(x, weight, dy, x_prev=None, want_dweight=True, want_dprev=False):
    """Returns (dx, dweight or None, dx_prev or None)."""
    B, T, D = _stream_shape(x)
    dx = torch.empty_like(x)
    dw = torch.empty((D, 4), dtype=torch.float32, device=x.device) if want_dweight else None
    dprev = torch.empty((B, 3, D), dtype=x.dtype, device=x.device) if want_dprev else None
    need = load().delta_rule_shortconv_workspace_size(B, T, D) if want_dweight else 0
    ws = _workspace(need, x.device) if need else None
    rc = shortconv_bwd_raw(_p(x), _p(weight), _p(x_prev), _p(dy), _p(dx), _p(dw), _p(dprev), B, T, D,
                           DTYPES[x.dtype], _p(ws), need, torch.cuda.current_stream(x.device).cuda_stream)
    _check(rc, "delta_rule_shortconv_bwd")
    return dx, dw, dprev


def clvr_raw(*args) -> int:
    return load().delta_rule_clvr(*args)


def clvr_bwd_raw(*args) -> int:
    return load().delta_rule_clvr_bwd(*args)


def delta_rule_clvr(u, W, h=None, out=None, workspace=None):
    """h + u W for write values u ([B, T, H, dv] or [M, K]) and W [K, N]; returns [..., N] shaped like h
    (or [M, N]).  out may be h itself (in-place residual add)."""
    K, N = W.shape
    M = u.numel() // K
    if out is None:
        out = torch.empty((M, N) if h is None else h.shape, dtype=u.dtype, device=u.device)
    need = load().delta_rule_clvr_workspace_size()
    ws = workspace if workspace is not None else _workspace(need, u.device)
    rc = clvr_raw(_p(u), _p(W), _p(h), _p(out), M, K, N, DTYPES[u.dtype], _p(ws), need,
                  torch.cuda.current_stream(u.device).cuda_stream)
    _check(rc, "delta_rule_clvr")
    return out


def delta_rule_clvr_bwd(u, W, dh_out, want_du=True, want_dW=True, workspace=None):
    """Returns (du shaped like u or None, dW [K, N] fp32 or None)."""
    K, N = W.shape
    M = u.numel() // K
    du = torch.empty_like(u) if want_du else None
    dW = torch.empty((K, N), dtype=torch.float32, device=u.device) if want_dW else None
    need = load().delta_rule_clvr_workspace_size()
    ws = workspace if workspace is not None else _workspace(need, u.device)
    rc = clvr_bwd_raw(_p(u), _p(W), _p(dh_out), _p(du), _p(dW), M, K, N, DTYPES[u.dtype], _p(ws), need,
                      torch.cuda.current_stream(u.device).cuda_stream)
    _check(rc, "delta_rule_clvr_bwd")
    return du, dW


def delta_rule_bwd(q, k, v, alpha, beta, S0, dout, du=None, dS_T=None, variant="gdn", chunk=64,
                   want_dS0=True, workspace: torch.Tensor | None = None, grads: dict | None = None):
    """Backward on CUDA tensors.  Returns dict(dq, dk, dv, dalpha (None for deltanet), dbeta, dS0)."""
    var = _variant(variant)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = DTYPES[q.dtype]
    dev = q.device
    g = dict(grads or {})
    g.setdefault("dq", torch.empty_like(q))
    g.setdefault("dk", torch.empty_like(k))
    g.setdefault("dv", torch.empty_like(v))
    g.setdefault("dalpha", torch.empty_like(alpha) if (var != DR_DELTANET and alpha is not None) else None)
    g.setdefault("dbeta", torch.empty_like(beta))
    g.setdefault("dS0", torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev) if want_dS0 else None)
    need = workspace_size(B, T, H, dk, dv, var, chunk, dt, 1)
    if workspace is None or workspace.numel() < need:
        workspace = _workspace(need, dev)
    stream = torch.cuda.current_stream(dev).cuda_stream
    rc = bwd_raw(_p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(S0), _p(dout), _p(du), _p(dS_T),
                 _p(g["dq"]), _p(g["dk"]), _p(g["dv"]), _p(g["dalpha"]), _p(g["dbeta"]), _p(g["dS0"]),
                 B, T, H, dk, dv, var, chunk, dt, _p(workspace), need, stream)
    _check(rc, "delta_rule_bwd")
    return g


def delta_rule_fwd_save(q, k, v, alpha, beta, S0=None, variant="gdn", chunk=64, want_u=True, want_state=True,
                        saved: torch.Tensor | None = None, workspace: torch.Tensor | None = None, out=None, u=None,
                        S_T=None):
    """The forward of a training step: returns (o, u or None, S_T or None, saved).

    ``saved`` (a uint8 CUDA tensor, allocated here when not given or too small) holds what
    ``delta_rule_bwd_saved`` needs instead of recomputing the forward; it is None for
    configurations without a saved form (then this is ``delta_rule_fwd``).
    """
    var = _variant(variant)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = DTYPES[q.dtype]
    dev = q.device
    out = torch.empty((B, T, H, dv), dtype=q.dtype, device=dev) if out is None else out
    if want_u and u is None:
        u = torch.empty((B, T, H, dv), dtype=q.dtype, device=dev)
    if want_state and S_T is None:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    sneed = saved_size(B, T, H, dk, dv, var, chunk, dt)
    if saved is None or saved.numel() < sneed:
        saved = _workspace(sneed, dev)
    need = workspace_size(B, T, H, dk, dv, var, chunk, dt, 2)
    if workspace is None or workspace.numel() < need:
        workspace = _workspace(need, dev)
    stream = torch.cuda.current_stream(dev).cuda_stream
    rc = fwd_save_raw(_p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(S0), _p(out), _p(u), _p(S_T),
                      B, T, H, dk, dv, var, chunk, dt, _p(saved), sneed, _p(workspace), need, stream)
    _check(rc, "delta_rule_fwd_save")
    return out, u, S_T, saved


def delta_rule_bwd_saved(q, k, v, alpha, beta, S0, dout, du=None, dS_T=None, saved=None, variant="gdn", chunk=64,
                         want_dS0=True, workspace: torch.Tensor | None = None, grads: dict | None = None):
    """The backward of a training step from ``saved`` (from ``delta_rule_fwd_save`` on the same inputs).

    Returns the same dict as ``delta_rule_bwd``.
    """
    var = _variant(variant)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = DTYPES[q.dtype]
    dev = q.device
    g = dict(grads or {})
    g.setdefault("dq", torch.empty_like(q))
    g.setdefault("dk", torch.empty_like(k))
    g.setdefault("dv", torch.empty_like(v))
    g.setdefault("dalpha", torch.empty_like(alpha) if (var != DR_DELTANET and alpha is not None) else None)
    g.setdefault("dbeta", torch.empty_like(beta))
    g.setdefault("dS0", torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev) if want_dS0 else None)
    sneed = saved_size(B, T, H, dk, dv, var, chunk, dt)
    need = workspace_size(B, T, H, dk, dv, var, chunk, dt, 3)
    if workspace is None or workspace.numel() < need:
        workspace = _workspace(need, dev)
    stream = torch.cuda.current_stream(dev).cuda_stream
    rc = bwd_saved_raw(_p(q), _p(k), _p(v), _p(alpha), _p(beta), _p(S0), _p(dout), _p(du), _p(dS_T),
                       _p(g["dq"]), _p(g["dk"]), _p(g["dv"]), _p(g["dalpha"]), _p(g["dbeta"]), _p(g["dS0"]),
                       B, T, H, dk, dv, var, chunk, dt, _p(saved), sneed, _p(workspace), need, stream)
    _check(rc, "delta_rule_bwd_saved")
    return g


def fwd_fused_raw(*args) -> int:
    return load().delta_rule_fwd_fused(*args)


def fused_workspace_size(B, T, H, dk, dv, variant, chunk, dtype) -> int:
    n = load().delta_rule_fwd_fused_workspace_size(B, T, H, dk, dv, variant, chunk, dtype)
    if n == ctypes.c_size_t(-1).value:
        raise DeltaRuleError(DR_ERR_UNSUPPORTED, "delta_rule_fwd_fused_workspace_size")
    return n


def delta_rule_fwd_fused(q_raw, k_raw, v, gate_raw, beta_raw, gate_out, w_norm, S0=None, variant="gdn", chunk=64,
                         want_o=False, want_u=True, want_state=True, workspace: torch.Tensor | None = None):
    """Pre-operation, forward and post-operation in the core's kernels: returns (y, o or None, u or None,
    S_T or None) for raw q, k projections and raw gate / beta logits (Gated DeltaNet, DeltaNet)."""
    var = _variant(variant)
    B, T, H, dk = q_raw.shape
    dv = v.shape[-1]
    dt = DTYPES[q_raw.dtype]
    dev = q_raw.device
    y = torch.empty((B, T, H, dv), dtype=q_raw.dtype, device=dev)
    o = torch.empty_like(y) if want_o else None
    u = torch.empty_like(y) if want_u else None
    S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev) if want_state else None
    need = fused_workspace_size(B, T, H, dk, dv, var, chunk, dt)
    if workspace is None or workspace.numel() < need:
        workspace = _workspace(need, dev)
    rc = fwd_fused_raw(_p(q_raw), _p(k_raw), _p(v), _p(gate_raw), _p(beta_raw), _p(S0), _p(gate_out), _p(w_norm),
                       _p(y), _p(o), _p(u), _p(S_T), B, T, H, dk, dv, var, chunk, dt, _p(workspace), need,
                       torch.cuda.current_stream(dev).cuda_stream)
    _check(rc, "delta_rule_fwd_fused")
    return y, o, u, S_T


def delta_rule_fwd_host(q, k, v, alpha, beta, S0=None, variant="gdn", chunk=64, device="cuda"):
    """The forward for host (CPU, ideally pinned) tensors: copy in, compute, copy out."""
    dev = torch.device(device)
    cp = [None if x is None else x.to(dev, non_blocking=True) for x in (q, k, v, alpha, beta, S0)]
    o, u, S = delta_rule_fwd(*cp, variant=variant, chunk=chunk)
    return o.to("cpu"), u.to("cpu"), S.to("cpu")
