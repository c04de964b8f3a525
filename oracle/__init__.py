"""fp64 CPU oracle for the gated delta rule -- TEST INFRASTRUCTURE ONLY.

This package is the independent checker for the CUDA library.  It shares no code
with ``gated_delta_rule_107_b200`` and is never imported by it.  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` may import it.

The arithmetic lives in ``delta_rule_oracle.c`` (plain C, double precision);
this module compiles it with gcc on first use and marshals numpy arrays.

What it computes -- the state update of "线性注意力架构演进与Kimi Delta Attention
创新实践" (Kimi Delta Attention page) section 2.1,
``S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T``,
``o_t = S_t^T q_t``, for DeltaNet (alpha == 1), Gated DeltaNet (scalar alpha per
token and head) and KDA (channel-wise alpha); plus the CLVR write value
``u_t = beta_t (v_t - (Diag(alpha_t) S_{t-1})^T k_t)`` ("线性注意力架构：机制、权衡
与跨层路由" explainer, "4. 跨层路由 CLVR").

Pins: every function here is checked by ``tests/test_oracle_pins.py`` against
closed forms, invariants, a hand-computed example (``tests/golden/``), a brute
force chunked solve and finite differences.  Nothing here is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

DELTANET, GATED, KDA = 0, 1, 2
VARIANTS = {"deltanet": DELTANET, "gdn": GATED, "gated": GATED, "kda": KDA}

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "delta_rule_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/liboracle.so`` (gcc, -O2, pthreads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-D_POSIX_C_SOURCE=200809L", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def load_library(path: str | None = None):
    """Load (building if needed) the oracle library; ``path`` loads another build of it."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
        return _lib


def _bind(lib):
    P = ctypes.POINTER(ctypes.c_double)
    i = ctypes.c_int
    lib.oracle_fwd.argtypes = [P] * 9 + [i] * 7
    lib.oracle_fwd.restype = i
    lib.oracle_bwd.argtypes = [P] * 15 + [i] * 7
    lib.oracle_bwd.restype = i
    lib.oracle_chunked_fwd.argtypes = [P] * 9 + [i] * 8
    lib.oracle_chunked_fwd.restype = i
    return lib


def _variant(v) -> int:
    return VARIANTS[v] if isinstance(v, str) else int(v)


def _in(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: widen the exact stored values
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(x):
    if x is None:
        return ctypes.POINTER(ctypes.c_double)()
    return x.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _dims(q, v):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    return B, T, H, dk, dv


def fwd(q, k, v, loga, beta, S0=None, variant="gdn", nthreads=0, lib=None):
    """Token-by-token recurrence.  Returns dict(o, u, S_T) as float64 arrays.

    q, k: [B,T,H,dk]; v: [B,T,H,dv]; loga: [B,T,H] (gdn) / [B,T,H,dk] (kda) /
    ignored (deltanet); beta: [B,T,H]; S0: [B,H,dk,dv] or None (zero).
    """
    lib = lib or load_library()
    q, k, v, loga, beta, S0 = map(_in, (q, k, v, loga, beta, S0))
    B, T, H, dk, dv = _dims(q, v)
    o = np.zeros((B, T, H, dv))
    u = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dk, dv))
    rc = lib.oracle_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(loga), _ptr(beta), _ptr(S0), _ptr(o), _ptr(u), _ptr(ST),
                        B, T, H, dk, dv, _variant(variant), nthreads)
    if rc:
        raise RuntimeError(f"oracle_fwd failed: {rc}")
    return {"o": o, "u": u, "S_T": ST}


def bwd(q, k, v, loga, beta, S0=None, dO=None, du=None, dS_T=None, variant="gdn", nthreads=0, lib=None):
    """Adjoint of :func:`fwd` for L = <dO,o> + <du,u> + <dS_T,S_T>.

    Returns dict(dq, dk, dv, dloga, dbeta, dS0) as float64 arrays (dloga has the
    shape of loga; it is all zeros for deltanet).
    """
    lib = lib or load_library()
    q, k, v, loga, beta, S0, dO, du, dS_T = map(_in, (q, k, v, loga, beta, S0, dO, du, dS_T))
    B, T, H, dk, dv = _dims(q, v)
    var = _variant(variant)
    dq = np.zeros_like(q)
    dk_ = np.zeros_like(k)
    dv_ = np.zeros_like(v)
    dl = np.zeros((B, T, H, dk) if var == KDA else (B, T, H))
    db = np.zeros((B, T, H))
    dS0 = np.zeros((B, H, dk, dv))
    rc = lib.oracle_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(loga), _ptr(beta), _ptr(S0), _ptr(dO), _ptr(du), _ptr(dS_T),
                        _ptr(dq), _ptr(dk_), _ptr(dv_), _ptr(dl), _ptr(db), _ptr(dS0),
                        B, T, H, dk, dv, var, nthreads)
    if rc:
        raise RuntimeError(f"oracle_bwd failed: {rc}")
    return {"dq": dq, "dk": dk_, "dv": dv_, "dloga": dl, "dbeta": db, "dS0": dS0}


def chunked_fwd(q, k, v, loga, beta, S0=None, variant="gdn", chunk=16, nthreads=0, lib=None):
    """Chunkwise (UT/WY) form solved by dense Gaussian elimination per chunk."""
    lib = lib or load_library()
    q, k, v, loga, beta, S0 = map(_in, (q, k, v, loga, beta, S0))
    B, T, H, dk, dv = _dims(q, v)
    o = np.zeros((B, T, H, dv))
    u = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dk, dv))
    rc = lib.oracle_chunked_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(loga), _ptr(beta), _ptr(S0), _ptr(o), _ptr(u),
                                _ptr(ST), B, T, H, dk, dv, _variant(variant), chunk, nthreads)
    if rc:
        raise RuntimeError(f"oracle_chunked_fwd failed: {rc}")
    return {"o": o, "u": u, "S_T": ST}
