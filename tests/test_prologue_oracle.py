"""Pins of the prologue oracle (oracle/prologue.py) to facts that do not come
from the oracle itself: closed forms of the normalisation and the gates,
library special functions (scipy), the forget gate as a plain power, and
central finite differences of the forward for the backward.  CPU only."""
import numpy as np
import pytest
import scipy.special as sp

from oracle import prologue as _P


def _inputs(seed, B=2, T=5, H=3, dk=4, dv=6):
    r = np.random.default_rng(seed)
    return dict(q_raw=r.normal(size=(B, T, H, dk)), k_raw=r.normal(size=(B, T, H, dk)),
                v_raw=r.normal(size=(B, T, H, dv)), beta_pre=r.normal(size=(B, T, H)) * 2,
                c_pre=r.normal(size=(B, T, H)) * 2, f_pre=r.normal(size=(B, T, H, dk)) * 3 + 2,
                a_log=r.normal(size=(H,)) * 0.5)


def test_l2_normalise_closed_form(P=_P):
    y, r = P.l2_normalise(np.array([[3.0, 4.0]]), eps=0.0)
    assert np.allclose(y, [[0.6, 0.8]], rtol=0, atol=1e-15)
    assert np.allclose(r, [[0.2]], rtol=0, atol=1e-15)
    # with eps the norm is sqrt(s / (s + eps)), slightly below one
    x = np.array([[1e-3, 0.0, 0.0]])
    y, _ = P.l2_normalise(x)
    assert np.isclose(np.linalg.norm(y), 1e-3 / np.sqrt(1e-6 + 1e-6), rtol=1e-12)
    # a zero row stays zero (no division by zero)
    y, _ = P.l2_normalise(np.zeros((1, 8)))
    assert np.all(y == 0)


def test_gates_match_library_special_functions(P=_P):
    x = np.linspace(-60, 60, 2001)
    assert np.allclose(P.sigmoid(x), sp.expit(x), rtol=1e-14, atol=0)
    assert np.allclose(P.log_sigmoid(x), sp.log_expit(x), rtol=1e-13, atol=1e-300)
    assert P.sigmoid(np.array([0.0]))[0] == 0.5
    assert np.isclose(P.log_sigmoid(np.array([0.0]))[0], -np.log(2.0), rtol=1e-15)
    # extreme arguments stay finite
    assert np.isfinite(P.log_sigmoid(np.array([-800.0, 800.0]))).all()


def test_forward_outputs_against_plain_definitions(P=_P):
    inp = _inputs(1)
    o = P.prologue_fwd(**inp, beta_scale=2.0)
    for n in ("q", "k", "v"):
        raw = inp[n + "_raw"]
        nrm = np.linalg.norm(raw, axis=-1, keepdims=True)
        assert np.allclose(o[n], raw / np.sqrt(nrm ** 2 + 1e-6), rtol=1e-13)
        assert (np.linalg.norm(o[n], axis=-1) < 1).all()
    assert np.allclose(o["beta"], 2.0 / (1.0 + np.exp(-inp["beta_pre"])), rtol=1e-13)
    assert ((o["beta"] > 0) & (o["beta"] < 2)).all()
    assert np.allclose(o["c"], 1.0 / (1.0 + np.exp(-inp["c_pre"])), rtol=1e-13)
    # the forget gate is sigmoid(x) raised to exp(a_log): f = sigma^a, logf <= 0
    a = np.exp(inp["a_log"])[None, None, :, None]
    f = (1.0 / (1.0 + np.exp(-inp["f_pre"]))) ** a
    assert np.allclose(np.exp(o["logf"]), f, rtol=1e-12)
    assert (o["logf"] <= 0).all()
    # a_log = 0 gives the plain sigmoid gate
    o0 = P.prologue_fwd(**{**inp, "a_log": np.zeros(3)})
    assert np.allclose(o0["logf"], np.log(sp.expit(inp["f_pre"])), rtol=1e-12)


def _loss(P, inp, w, beta_scale):
    o = P.prologue_fwd(**inp, beta_scale=beta_scale)
    return sum(float(np.sum(w[n] * o[n])) for n in o)


@pytest.mark.parametrize("beta_scale", [1.0, 2.0])
def test_backward_matches_central_differences(beta_scale, P=_P):
    inp = _inputs(2)
    r = np.random.default_rng(7)
    o = P.prologue_fwd(**inp, beta_scale=beta_scale)
    w = {n: r.normal(size=o[n].shape) for n in o}
    g = P.prologue_bwd(**inp, dq=w["q"], dk=w["k"], dv=w["v"], dbeta=w["beta"], dc=w["c"],
                       dlogf=w["logf"], beta_scale=beta_scale)
    names = dict(q_raw="dq_raw", k_raw="dk_raw", v_raw="dv_raw", beta_pre="dbeta_pre", c_pre="dc_pre",
                 f_pre="df_pre", a_log="da_log")
    h = 1e-6
    for x, gname in names.items():
        fd = np.zeros_like(inp[x])
        flat = inp[x].reshape(-1)
        for i in range(flat.size):
            keep = flat[i]
            flat[i] = keep + h
            lp = _loss(P, inp, w, beta_scale)
            flat[i] = keep - h
            lm = _loss(P, inp, w, beta_scale)
            flat[i] = keep
            fd.reshape(-1)[i] = (lp - lm) / (2 * h)
        assert np.allclose(g[gname], fd, rtol=1e-6, atol=1e-7), x


def test_prologue_then_recurrence_gradient(P=_P):
    """The prologue's backward chained after the recurrence's (fp64 oracle)
    matches central differences of the composite on a tiny problem."""
    from oracle import oracle as O
    inp = _inputs(3, B=1, T=4, H=2, dk=3, dv=2)
    r = np.random.default_rng(11)
    dO = r.normal(size=(1, 4, 2, 2))

    def loss(x):
        o = P.prologue_fwd(**x)
        out, _ = O.fwd(o["q"], o["k"], o["v"], o["beta"], o["c"], o["logf"])
        return float(np.sum(dO * out))

    o = P.prologue_fwd(**inp)
    g = O.bwd(o["q"], o["k"], o["v"], o["beta"], o["c"], o["logf"], None, dO, None)
    gp = P.prologue_bwd(**inp, dq=g["dq"], dk=g["dk"], dv=g["dv"], dbeta=g["dbeta"], dc=g["dc"],
                        dlogf=g["dlogf"])
    h = 1e-6
    for x, gname in (("q_raw", "dq_raw"), ("v_raw", "dv_raw"), ("f_pre", "df_pre"), ("a_log", "da_log"),
                     ("beta_pre", "dbeta_pre")):
        flat = inp[x].reshape(-1)
        fd = np.zeros(flat.size)
        for i in range(flat.size):
            keep = flat[i]
            flat[i] = keep + h
            lp = loss(inp)
            flat[i] = keep - h
            lm = loss(inp)
            flat[i] = keep
            fd[i] = (lp - lm) / (2 * h)
        assert np.allclose(gp[gname].reshape(-1), fd, rtol=1e-5, atol=1e-8), x


# (name, exact text in prologue.py, replacement): plausible mistakes, each of
# which one of the pins above must reject
MUTANTS = [
    ("norm-no-sqrt", "r = 1.0 / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)",
     "r = 1.0 / (np.sum(x * x, axis=-1, keepdims=True) + eps)"),
    ("norm-no-eps", "keepdims=True) + eps)", "keepdims=True))"),
    ("beta-unscaled", "beta = beta_scale * sigmoid(beta_pre)", "beta = sigmoid(beta_pre)"),
    ("forget-no-exponent", "    logf = a[None, None, :, None] * log_sigmoid(f_pre)\n    return dict",
     "    logf = log_sigmoid(f_pre)\n    return dict"),
    ("log-sigmoid-sign", "np.maximum(-x, 0.0)", "np.maximum(x, 0.0)"),
    ("dx-sign", "r * (g - y * np.sum", "r * (g + y * np.sum"),
    ("dx-no-projection", "out[name] = r * (g - y * np.sum(y * g, axis=-1, keepdims=True))",
     "out[name] = r * g"),
    ("dbeta-unscaled", "_f64(dbeta) * beta_scale * sigmoid", "_f64(dbeta) * sigmoid"),
    ("df-missing-exponent", "dlogf * a[None, None, :, None] * sigmoid(-_f64(f_pre))",
     "dlogf * sigmoid(-_f64(f_pre))"),
    ("df-sigma-not-complement", "* sigmoid(-_f64(f_pre))", "* sigmoid(f_pre)"),
    ("dc-one-factor", "_f64(dc) * sigmoid(c_pre) * sigmoid(-_f64(c_pre))", "_f64(dc) * sigmoid(c_pre)"),
    ("dalog-missing-logf", "np.sum(dlogf * logf, axis=(0, 1, 3))", "np.sum(dlogf, axis=(0, 1, 3))"),
]


def _mutant(tmp_path, name, old, new):
    import importlib.util
    src = open(_P.__file__).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    f = tmp_path / f"prologue_{name.replace('-', '_')}.py"
    f.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location(f.stem, f)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_reject_mutant(tmp_path, name, old, new):
    M = _mutant(tmp_path, name, old, new)
    pins = [lambda: test_l2_normalise_closed_form(M), lambda: test_gates_match_library_special_functions(M),
            lambda: test_forward_outputs_against_plain_definitions(M),
            lambda: test_backward_matches_central_differences(2.0, M)]
    caught = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught > 0, f"no pin rejects mutant {name}"


def test_backward_tails_are_accurate(P=_P):
    """In the saturated tails the gate derivatives keep their relative accuracy:
    d/dx log sigmoid(x) = sigmoid(-x) ~ e^-x and sigmoid'(x) ~ e^-|x| (closed forms)."""
    x = np.array([30.0, -30.0, 60.0])
    z = np.zeros((1, 1, 1, 3))
    g = P.prologue_bwd(z + 1, z + 1, z[..., :1] + 1, x.reshape(1, 1, 3)[..., :1].reshape(1, 1, 1),
                       np.array([[[40.0]]]), x.reshape(1, 1, 1, 3), np.zeros(1),
                       z, z, z[..., :1], np.ones((1, 1, 1)), np.ones((1, 1, 1)), np.ones((1, 1, 1, 3)))
    assert np.allclose(g["df_pre"].reshape(-1), [np.exp(-30.0) / (1 + np.exp(-30.0)),
                                                  1.0 / (1.0 + np.exp(-30.0)), np.exp(-60.0)], rtol=1e-12)
    assert np.isclose(g["dc_pre"].item(), np.exp(-40.0), rtol=1e-12)
    assert np.isclose(g["dbeta_pre"].item(), np.exp(-30.0), rtol=1e-12)
