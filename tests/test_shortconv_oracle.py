"""Pins of the short-convolution oracle (oracle/shortconv.py) against numpy's own convolution,
the identity and one-token-shift filters, splitting a stream across calls through the cache,
and central finite differences of the backward.  Planted mistakes in copies of the oracle's
source must each fail at least one pin."""
import types

import numpy as np
import pytest

from oracle import shortconv as SC


def _rng():
    return np.random.default_rng(77)


def pin_numpy_convolve(sc):
    rng = _rng()
    B, T, D = 2, 19, 5
    x, w, prev = rng.standard_normal((B, T, D)), rng.standard_normal((D, 4)), rng.standard_normal((B, 3, D))
    for x_prev in (None, prev):
        y, _ = sc.shortconv_fwd(x, w, x_prev)
        for b in range(B):
            for c in range(D):
                head = np.zeros(3) if x_prev is None else x_prev[b, :, c]
                seq = np.concatenate([head, x[b, :, c]])
                # numpy's convolution flips its second operand, so the taps go in reversed
                ref = np.convolve(seq, w[c, ::-1], mode="valid")
                assert np.allclose(y[b, :, c], ref, atol=1e-12)


def pin_identity_and_shift(sc):
    rng = _rng()
    B, T, D = 2, 7, 3
    x, prev = rng.standard_normal((B, T, D)), rng.standard_normal((B, 3, D))
    ident = np.tile([0.0, 0.0, 0.0, 1.0], (D, 1))
    shift = np.tile([0.0, 0.0, 1.0, 0.0], (D, 1))
    assert np.array_equal(sc.shortconv_fwd(x, ident, prev)[0], x)
    y, cache = sc.shortconv_fwd(x, shift, prev)
    assert np.array_equal(y[:, 1:], x[:, :-1]) and np.array_equal(y[:, 0], prev[:, 2])
    assert np.array_equal(sc.shortconv_fwd(x, shift)[0][:, 0], np.zeros((B, D)))
    assert np.array_equal(cache, x[:, -3:])


def pin_stream_split(sc):
    rng = _rng()
    B, T, D = 2, 23, 4
    x, w = rng.standard_normal((B, T, D)), rng.standard_normal((D, 4))
    whole, cache = sc.shortconv_fwd(x, w)
    parts, c = [], None
    for a, b in ((0, 1), (1, 3), (3, 10), (10, 23)):  # pieces shorter than the cache too
        y, c = sc.shortconv_fwd(x[:, a:b], w, c)
        parts.append(y)
    assert np.allclose(np.concatenate(parts, axis=1), whole, atol=1e-13)
    assert np.array_equal(c, cache)
    y0, c0 = sc.shortconv_fwd(x[:, :0], w, cache)  # an empty piece leaves the cache as it was
    assert y0.shape == (B, 0, D) and np.array_equal(c0, cache)


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


def pin_backward_finite_differences(sc):
    rng = _rng()
    B, T, D = 2, 6, 3
    x, w, prev = rng.standard_normal((B, T, D)), rng.standard_normal((D, 4)), rng.standard_normal((B, 3, D))
    dy = rng.standard_normal((B, T, D))

    def loss(x_, w_, p_):
        return np.sum(SC.shortconv_fwd(x_, w_, p_)[0] * dy)  # the pinned forward

    got = sc.shortconv_bwd(x, w, dy, prev)
    assert np.allclose(got["dx"], _fd(lambda t: loss(t, w, prev), x), atol=1e-8)
    assert np.allclose(got["dw"], _fd(lambda t: loss(x, t, prev), w), atol=1e-8)
    assert np.allclose(got["dx_prev"], _fd(lambda t: loss(x, w, t), prev), atol=1e-8)
    got0 = sc.shortconv_bwd(x, w, dy)  # without a cache the leading tokens read zeros
    assert np.allclose(got0["dw"], _fd(lambda t: loss(x, t, None), w), atol=1e-8)


PINS = [pin_numpy_convolve, pin_identity_and_shift, pin_stream_split, pin_backward_finite_differences]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(SC)


MUTANTS = [
    ("taps_reversed", "y += w[:, j] * xp[:, j:j + T]", "y += w[:, K - 1 - j] * xp[:, j:j + T]"),
    ("cache_ignored", "prev = np.zeros((B, K - 1, D)) if x_prev is None else _f64(x_prev)",
     "prev = np.zeros((B, K - 1, D))"),
    ("old_cache_returned", "return y, xp[:, T:].copy()", "return y, xp[:, :K - 1].copy()"),
    ("bwd_dx_taps_reversed", "dxp[:, j:j + T] += w[:, j] * dy", "dxp[:, j:j + T] += w[:, K - 1 - j] * dy"),
    ("bwd_dw_tap_index", "dw[:, j] = np.sum(dy * xp[:, j:j + T], axis=(0, 1))",
     "dw[:, K - 1 - j] = np.sum(dy * xp[:, j:j + T], axis=(0, 1))"),
    ("bwd_cache_grad_dropped", '"dx_prev": dxp[:, :K - 1]', '"dx_prev": 0 * dxp[:, :K - 1]'),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new):
    src = open(SC.__file__).read()
    assert src.count(old) == 1, f"mutation site for {name}"
    mod = types.ModuleType(f"shortconv_{name}")
    exec(compile(src.replace(old, new), f"<{name}>", "exec"), mod.__dict__)
    caught = 0
    for pin in PINS:
        try:
            pin(mod)
        except AssertionError:
            caught += 1
    assert caught > 0, f"no pin catches {name}"
