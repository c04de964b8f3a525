"""Pins of the routing oracle (oracle/clvr.py): a zero projection leaves the hidden stream
exactly as it was (the zero initialisation) while its gradient is already nonzero, a projection
with a single unit entry copies one write-value channel into one hidden channel, the four-
dimensional write-value layout equals its flattened matrix, and central finite differences of
the backward.  Planted mistakes in copies of the source must each fail a pin."""
import types

import numpy as np
import pytest

from oracle import clvr as CL


def _rng():
    return np.random.default_rng(91)


def pin_zero_projection_is_identity(cl):
    rng = _rng()
    u, h, dh = rng.standard_normal((7, 6)), rng.standard_normal((7, 5)), rng.standard_normal((7, 5))
    W0 = np.zeros((6, 5))
    assert np.array_equal(cl.clvr_fwd(u, W0, h), h)
    g = cl.clvr_bwd(u, W0, dh)
    assert np.array_equal(g["du"], np.zeros((7, 6)))
    assert np.abs(g["dW"]).max() > 0  # the zero-initialised projection still receives a gradient


def pin_unit_entry_routes_one_channel(cl):
    rng = _rng()
    u, h = rng.standard_normal((9, 6)), rng.standard_normal((9, 5))
    for i, j in ((0, 0), (5, 2), (3, 4)):
        W = np.zeros((6, 5))
        W[i, j] = 1.0
        out = cl.clvr_fwd(u, W, h)
        want = h.copy()
        want[:, j] += u[:, i]
        assert np.array_equal(out, want)
    assert np.array_equal(cl.clvr_fwd(u, 2.5 * np.eye(6, 5)), 2.5 * u[:, :5])  # no h: a zero stream


def pin_head_layout(cl):
    rng = _rng()
    u4 = rng.standard_normal((2, 3, 4, 2))  # [B, T, H, dv]: K = 8
    W, h = rng.standard_normal((8, 5)), rng.standard_normal((6, 5))
    flat = u4.reshape(6, 8)
    assert np.allclose(cl.clvr_fwd(u4, W, h), cl.clvr_fwd(flat, W, h), atol=0)
    # each row of the result depends only on its own token
    out = cl.clvr_fwd(flat, W, h)
    flat2 = flat.copy()
    flat2[3] += 1.0
    assert np.array_equal(cl.clvr_fwd(flat2, W, h)[[0, 1, 2, 4, 5]], out[[0, 1, 2, 4, 5]])


def _fd(f, x, h=1e-6):
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        xp, xm = x.copy(), x.copy()
        xp[i] += h
        xm[i] -= h
        g[i] = (f(xp) - f(xm)) / (2 * h)
    return g


def pin_backward_finite_differences(cl):
    rng = _rng()
    u, W, h, dh = (rng.standard_normal(s) for s in ((5, 4), (4, 3), (5, 3), (5, 3)))
    g = cl.clvr_bwd(u, W, dh)
    assert np.allclose(g["du"], _fd(lambda t: np.sum(CL.clvr_fwd(t, W, h) * dh), u), atol=1e-8)
    assert np.allclose(g["dW"], _fd(lambda t: np.sum(CL.clvr_fwd(u, t, h) * dh), W), atol=1e-8)


PINS = [pin_zero_projection_is_identity, pin_unit_entry_routes_one_channel, pin_head_layout,
        pin_backward_finite_differences]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(CL)


MUTANTS = [
    ("residual_dropped", "        out = out + _f64(h).reshape(out.shape)", "        out = out"),
    ("projection_transposed", "    out = U @ W\n", "    out = U @ W.T\n"),
    ("du_without_transpose", '"du": dH @ W.T', '"du": dH @ W'),
    ("dW_operands_swapped", '"dW": U.T @ dH', '"dW": dH.T @ U'),
    ("dW_missing", '"dW": U.T @ dH', '"dW": 0 * (U.T @ dH)'),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new):
    src = open(CL.__file__).read()
    assert src.count(old) == 1, f"mutation site for {name}"
    mod = types.ModuleType(f"clvr_{name}")
    exec(compile(src.replace(old, new), f"<{name}>", "exec"), mod.__dict__)
    caught = 0
    for pin in PINS:
        try:
            pin(mod)
        except (AssertionError, ValueError):
            caught += 1
    assert caught > 0, f"no pin catches {name}"
