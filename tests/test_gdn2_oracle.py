"""Pins of the Gated DeltaNet-2 oracle (oracle/gdn2.py) to facts that do not
come from the oracle: the special cases the article names (section "핵심 기여":
b = w = beta*1 gives the KDA-style gated delta rule, no erase gives gated
linear attention), the write hitting its target, a one-channel key reducing to
a scalar recursion written out by hand, a brute-force product of transition
matrices, central finite differences, and planted mistakes.  CPU only."""
import numpy as np
import pytest

from oracle import gdn2 as _G


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _inputs(seed, B=1, T=6, H=2, dk=4, dv=3, s0=True):
    r = np.random.default_rng(seed)
    return dict(q=_unit(r.normal(size=(B, T, H, dk))), k=_unit(r.normal(size=(B, T, H, dk))),
                v=_unit(r.normal(size=(B, T, H, dv))), b=r.uniform(0.1, 1.0, size=(B, T, H, dk)),
                w=r.uniform(0.1, 1.0, size=(B, T, H, dv)), loga=-r.uniform(0.0, 0.5, size=(B, T, H, dk)),
                S0=r.normal(size=(B, H, dv, dk)) * 0.3 if s0 else None)


def test_full_erase_and_write_hits_the_target(G=_G):
    """b = w = 1, unit keys: after the write S_t k_t = v_t exactly."""
    x = _inputs(1, T=1)
    x["b"][:] = 1.0
    x["w"][:] = 1.0
    O, S = G.fwd(**x)
    assert np.allclose(np.einsum("bhrj,bhj->bhr", S, x["k"][:, 0]), x["v"][:, 0], atol=1e-14)


def test_no_erase_is_gated_linear_attention(G=_G):
    """b = 0: S_T = S0 Gamma_T + sum_i (w_i o v_i) (k_i o gamma_T/gamma_i)^T and
    o_t = S_t q_t, written as sums over tokens."""
    x = _inputs(2, T=7)
    x["b"][:] = 0.0
    O, S = G.fwd(**x)
    L = np.cumsum(x["loga"], axis=1)
    z = x["w"] * x["v"]
    for t in range(7):
        St = x["S0"] * np.exp(L[:, t])[:, :, None, :]
        for i in range(t + 1):
            St = St + z[:, i][..., :, None] * (x["k"][:, i] * np.exp(L[:, t] - L[:, i]))[..., None, :]
        assert np.allclose(O[:, t], np.einsum("bhrj,bhj->bhr", St, x["q"][:, t]), atol=1e-13)
    assert np.allclose(S, St, atol=1e-13)


def test_scalar_key_recursion(G=_G):
    """dk = 1, k_t = kappa_t (a scalar): s_t = a_t s_{t-1} (1 - b_t kappa_t^2) + kappa_t w_t v_t."""
    r = np.random.default_rng(3)
    T, dv = 9, 3
    kap = r.uniform(-1, 1, size=T)
    x = dict(q=r.normal(size=(1, T, 1, 1)), k=kap.reshape(1, T, 1, 1), v=r.normal(size=(1, T, 1, dv)),
             b=r.uniform(0, 1, size=(1, T, 1, 1)), w=r.uniform(0, 1, size=(1, T, 1, dv)),
             loga=-r.uniform(0, 1, size=(1, T, 1, 1)), S0=r.normal(size=(1, 1, dv, 1)))
    O, S = G.fwd(**x)
    s = x["S0"][0, 0, :, 0].copy()
    for t in range(T):
        a = np.exp(x["loga"][0, t, 0, 0])
        s = a * s * (1.0 - x["b"][0, t, 0, 0] * kap[t] ** 2) + kap[t] * x["w"][0, t, 0] * x["v"][0, t, 0]
        assert np.allclose(O[0, t, 0], s * x["q"][0, t, 0, 0], atol=1e-14)
    assert np.allclose(S[0, 0, :, 0], s, atol=1e-14)


def test_transition_matrix_product(G=_G):
    """S_t = S_{t-1} D_t (I - e_t k_t^T) + z_t k_t^T, composed as explicit dk x dk matrices."""
    x = _inputs(4, T=5, dk=5, dv=2)
    O, S = G.fwd(**x)
    for bh in range(2):
        St = x["S0"][0, bh]
        for t in range(5):
            k, e = x["k"][0, t, bh], x["b"][0, t, bh] * x["k"][0, t, bh]
            M = np.diag(np.exp(x["loga"][0, t, bh])) @ (np.eye(5) - np.outer(e, k))
            St = St @ M + np.outer(x["w"][0, t, bh] * x["v"][0, t, bh], k)
        assert np.allclose(S[0, bh], St, atol=1e-13)


def test_gated_delta_rule_special_case(G=_G):
    """b = w = beta*1: S_t = Sbar + beta (v - Sbar k) k^T, the gated delta rule
    (KDA with a channel-wise decay)."""
    x = _inputs(5, T=6)
    beta = np.random.default_rng(6).uniform(0.2, 1.0, size=(1, 6, 2))
    x["b"] = np.repeat(beta[..., None], 4, axis=-1)
    x["w"] = np.repeat(beta[..., None], 3, axis=-1)
    O, S = G.fwd(**x)
    St = x["S0"].copy()
    for t in range(6):
        Sbar = St * np.exp(x["loga"][:, t])[:, :, None, :]
        pred = np.einsum("bhrj,bhj->bhr", Sbar, x["k"][:, t])
        St = Sbar + (beta[:, t][..., None] * (x["v"][:, t] - pred))[..., :, None] * x["k"][:, t][..., None, :]
        assert np.allclose(O[:, t], np.einsum("bhrj,bhj->bhr", St, x["q"][:, t]), atol=1e-13)


def test_backward_matches_central_differences(G=_G):
    x = _inputs(7, T=5, dk=3, dv=2)
    r = np.random.default_rng(8)
    dO = r.normal(size=(1, 5, 2, 2))
    dST = r.normal(size=(1, 2, 2, 3))

    def loss():
        O, S = G.fwd(**x)
        return float(np.sum(dO * O) + np.sum(dST * S))

    g = G.bwd(**x, dO=dO, dST=dST)
    h = 1e-6
    for n in ("q", "k", "v", "b", "w", "loga", "S0"):
        flat = x[n].reshape(-1)
        fd = np.zeros(flat.size)
        for i in range(flat.size):
            keep = flat[i]
            flat[i] = keep + h
            lp = loss()
            flat[i] = keep - h
            lm = loss()
            flat[i] = keep
            fd[i] = (lp - lm) / (2 * h)
        assert np.allclose(g["d" + n].reshape(-1), fd, rtol=1e-6, atol=1e-8), n


MUTANTS = [
    ("erase-sign", "u = w[:, t] * v[:, t] - np.einsum(\"bhrj,bhj->bhr\", Sbar, e)\n        S = Sbar + u[..., :, None] * k[:, t][..., None, :]\n        O[:, t]",
     "u = w[:, t] * v[:, t] + np.einsum(\"bhrj,bhj->bhr\", Sbar, e)\n        S = Sbar + u[..., :, None] * k[:, t][..., None, :]\n        O[:, t]"),
    ("erase-without-gate", "        e = b[:, t] * k[:, t]\n        u = w[:, t] * v[:, t] - np.einsum(\"bhrj,bhj->bhr\", Sbar, e)\n        S = Sbar + u[..., :, None] * k[:, t][..., None, :]\n        O[:, t]",
     "        e = k[:, t]\n        u = w[:, t] * v[:, t] - np.einsum(\"bhrj,bhj->bhr\", Sbar, e)\n        S = Sbar + u[..., :, None] * k[:, t][..., None, :]\n        O[:, t]"),
    ("decay-after-erase-read", "        Sbar = S * np.exp(loga[:, t])[:, :, None, :]\n        e = b[:, t] * k[:, t]\n        u = w[:, t] * v[:, t] - np.einsum(\"bhrj,bhj->bhr\", Sbar, e)\n        S = Sbar + u[..., :, None] * k[:, t][..., None, :]\n        O[:, t]",
     "        Sbar = S * np.exp(loga[:, t])[:, :, None, :]\n        e = b[:, t] * k[:, t]\n        u = w[:, t] * v[:, t] - np.einsum(\"bhrj,bhj->bhr\", S, e)\n        S = Sbar + u[..., :, None] * k[:, t][..., None, :]\n        O[:, t]"),
    ("write-transposed", "        S = Sbar + u[..., :, None] * k[:, t][..., None, :]\n        O[:, t]",
     "        S = Sbar + (u[..., :, None] * k[:, t][..., None, :])[..., ::-1, ::-1]\n        O[:, t]"),
    ("bwd-dk-missing-erase", "out[\"dk\"][:, t] = dk_t + de * bt", "out[\"dk\"][:, t] = dk_t"),
    ("bwd-dloga-after-erase", "out[\"dloga\"][:, t] = np.einsum(\"bhrj,bhrj->bhj\", dSbar, Sbar)",
     "out[\"dloga\"][:, t] = np.einsum(\"bhrj,bhrj->bhj\", G, Sbar)"),
    ("bwd-dq-prev-state", "out[\"dq\"][:, t] = np.einsum(\"bhrj,bhr->bhj\", St, dO[:, t])",
     "out[\"dq\"][:, t] = np.einsum(\"bhrj,bhr->bhj\", Sprev, dO[:, t])"),
    ("bwd-no-state-decay", "G = dSbar * D[:, :, None, :]", "G = dSbar"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_reject_mutant(tmp_path, name, old, new):
    import importlib.util
    src = open(_G.__file__).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    f = tmp_path / f"gdn2_{name.replace('-', '_')}.py"
    f.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location(f.stem, f)
    M = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(M)
    caught = 0
    for pin in (test_full_erase_and_write_hits_the_target, test_no_erase_is_gated_linear_attention,
                test_scalar_key_recursion, test_transition_matrix_product, test_gated_delta_rule_special_case,
                test_backward_matches_central_differences):
        try:
            pin(M)
        except (AssertionError, ValueError):
            caught += 1
    assert caught > 0, f"no pin rejects mutant {name}"
