"""Pins of the pre/post-operation oracle (oracle/prepost.py) against properties the
definitions fix: unit norm and scale invariance of the L2 normalisation, the symmetries
of the logistic gates, the RMS of the normalised output, and central finite differences
of every backward."""
import numpy as np
import pytest

from oracle import prepost as pp

RNG = np.random.default_rng(2024)


def test_l2norm_gives_unit_rows_and_is_scale_invariant():
    x = RNG.standard_normal((3, 5, 2, 128)) * 7.0
    y = pp.l2norm_fwd(x)
    assert np.allclose(np.linalg.norm(y, axis=-1), 1.0, atol=1e-7)
    assert np.allclose(pp.l2norm_fwd(3.5 * x), y, atol=1e-8)
    assert np.allclose(pp.l2norm_fwd(-x), -y)
    # the direction is kept: y is a positive multiple of x
    assert np.all(np.sum(y * x, axis=-1) > 0) and np.allclose(np.abs(np.sum(y * x, axis=-1)),
                                                              np.linalg.norm(x, axis=-1), rtol=1e-7)


def test_zero_row_stays_finite():
    assert np.all(pp.l2norm_fwd(np.zeros((1, 64))) == 0.0)
    assert np.all(np.isfinite(pp.postop_fwd(np.zeros((2, 64)), np.zeros((2, 64)))))


def test_logistic_gate_symmetries():
    b = RNG.standard_normal(1000) * 6
    out_p, out_m = pp.preop_fwd(np.ones((1, 4)), np.ones((1, 4)), b, b), pp.preop_fwd(np.ones((1, 4)),
                                                                                      np.ones((1, 4)), -b, -b)
    assert np.allclose(out_p["beta"] + out_m["beta"], 1.0)                  # sigmoid(x) + sigmoid(-x) = 1
    assert np.allclose(out_p["loga"] - out_m["loga"], -b, atol=1e-12)     # log-sigmoid(-x) - log-sigmoid(x) = -x
    assert np.all(out_p["loga"] < 0) and np.all((out_p["beta"] > 0) & (out_p["beta"] < 1))
    z = pp.preop_fwd(np.ones((1, 4)), np.ones((1, 4)), np.zeros(1), np.zeros(1))
    assert z["beta"][0] == 0.5 and abs(z["loga"][0] + np.log(2.0)) < 1e-15
    # a forget logit of -3 keeps about 95 % of the state per token (the -3 forget-gate bias of the Kimi Delta Attention page, section 7.1)
    assert abs(np.exp(pp.preop_fwd(np.ones((1, 4)), np.ones((1, 4)), np.zeros(1), np.array([-3.0]))["loga"][0])
               - 1 / (1 + np.exp(-3.0))) < 1e-15
    # extreme logits stay finite
    big = pp.preop_fwd(np.ones((1, 4)), np.ones((1, 4)), np.array([800.0, -800.0]), np.array([800.0, -800.0]))
    assert np.all(np.isfinite(big["beta"])) and np.all(np.isfinite(big["loga"]))
    assert big["loga"][0] == -800.0 and big["loga"][1] == 0.0


def test_rmsnorm_output_has_the_weights_rms():
    o = RNG.standard_normal((4, 3, 2, 128)) * 3.0
    g = np.full(o.shape, 40.0)  # sigmoid(g) = 1 to double precision
    y = pp.postop_fwd(o, g)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, atol=1e-6)
    assert np.allclose(pp.postop_fwd(5.0 * o, g), y, atol=1e-7)            # scale invariance
    w = RNG.standard_normal(128)
    assert np.allclose(pp.postop_fwd(o, np.zeros(o.shape), w), 0.5 * y * w, atol=1e-7)  # gate 0 halves


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


@pytest.mark.parametrize("gated", (True, False))
def test_preop_backward_matches_finite_differences(gated):
    q, k = RNG.standard_normal((2, 3, 2, 8)), RNG.standard_normal((2, 3, 2, 8))
    b = RNG.standard_normal((2, 3, 2))
    a = RNG.standard_normal((2, 3, 2)) if gated else None
    dq, dk = RNG.standard_normal(q.shape), RNG.standard_normal(k.shape)
    db, da = RNG.standard_normal(b.shape), RNG.standard_normal(b.shape)

    def loss(q_, k_, b_, a_):
        r = pp.preop_fwd(q_, k_, b_, a_)
        s = np.sum(r["q"] * dq) + np.sum(r["k"] * dk) + np.sum(r["beta"] * db)
        return s + (np.sum(r["loga"] * da) if a_ is not None else 0.0)

    got = pp.preop_bwd(q, k, b, a, dq, dk, db, da)
    assert np.allclose(got["dq"], _fd(lambda x: loss(x, k, b, a), q), atol=1e-7)
    assert np.allclose(got["dk"], _fd(lambda x: loss(q, x, b, a), k), atol=1e-7)
    assert np.allclose(got["db"], _fd(lambda x: loss(q, k, x, a), b), atol=1e-7)
    if gated:
        assert np.allclose(got["da"], _fd(lambda x: loss(q, k, b, x), a), atol=1e-7)
    else:
        assert got["da"] is None


def test_postop_backward_matches_finite_differences():
    o, g = RNG.standard_normal((2, 3, 2, 8)), RNG.standard_normal((2, 3, 2, 8))
    w, dy = RNG.standard_normal(8), RNG.standard_normal((2, 3, 2, 8))

    def loss(o_, g_, w_):
        return np.sum(pp.postop_fwd(o_, g_, w_) * dy)

    got = pp.postop_bwd(o, g, w, dy)
    assert np.allclose(got["do"], _fd(lambda x: loss(x, g, w), o), atol=1e-7)
    assert np.allclose(got["dg"], _fd(lambda x: loss(o, x, w), g), atol=1e-7)
    assert np.allclose(got["dw"], _fd(lambda x: loss(o, g, x), w), atol=1e-7)


# ---- planted mistakes in copies of the oracle's source must each fail a pin above ----
import types  # noqa: E402

PINS = [test_l2norm_gives_unit_rows_and_is_scale_invariant, test_zero_row_stays_finite, test_logistic_gate_symmetries,
        test_rmsnorm_output_has_the_weights_rms, lambda: test_preop_backward_matches_finite_differences(True),
        lambda: test_preop_backward_matches_finite_differences(False),
        test_postop_backward_matches_finite_differences]

MUTANTS = [
    ("l2norm_sum_not_root", "return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + EPS)",
     "return x / (np.sum(x * x, axis=-1, keepdims=True) + EPS)"),
    ("l2norm_bwd_projection_dropped", "return (dy - y * np.sum(y * dy, axis=-1, keepdims=True)) / r", "return dy / r"),
    ("beta_grad_without_derivative", '"db": _f64(dbeta) * beta * (1.0 - beta)', '"db": _f64(dbeta) * beta'),
    ("gate_grad_sign", 'out["da"] = -_f64(dloga) * _sigmoid(_f64(a))', 'out["da"] = _f64(dloga) * _sigmoid(_f64(a))'),
    ("softplus_sign", '"loga": None if a is None else -_softplus(a)}', '"loga": None if a is None else _softplus(a)}'),
    ("rms_sum_not_mean", "n = o / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + EPS)",
     "n = o / np.sqrt(np.sum(o * o, axis=-1, keepdims=True) + EPS)"),
    ("postop_dw_without_n", "dw = np.sum((dz * n).reshape(-1, d), axis=0)", "dw = np.sum(dz.reshape(-1, d), axis=0)"),
    ("postop_do_projection_dropped", "do = r * (dn - n * np.mean(dn * n, axis=-1, keepdims=True))", "do = r * dn"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new, monkeypatch):
    src = open(pp.__file__).read()
    assert src.count(old) == 1, f"mutation site for {name}"
    mod = types.ModuleType(f"prepost_{name}")
    exec(compile(src.replace(old, new), f"<{name}>", "exec"), mod.__dict__)
    monkeypatch.setitem(globals(), "pp", mod)  # the pins above read the module through this name
    caught = 0
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught > 0, f"no pin catches {name}"
