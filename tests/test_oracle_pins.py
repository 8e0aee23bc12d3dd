"""Pins for the fp64 oracle: facts the pages and the mathematics fix.

Sources: the KronLSTM digest ("KronLSTM이 스칼라 보정으로 긴 문맥 선형 어텐션의
기억 간섭을 줄인다"), sections "어떻게 동작하나" (erase/write split), "무엇과
다른가" (vectorised Widrow-Hoff form, interference, capacity) and "어떻게 쓰나"
(right-side key-channel decay, non-expansive updates); the Gated DeltaNet-2
article, section "핵심 기여" (KDA as a special case of the gated delta rules).

Each check uses an independent formula (Kronecker-vectorised transition
matrices, gated linear attention closed form, the KDA recurrence written in
the transposed convention, finite differences) so that a dropped term, a sign
error or a transposed operand in the oracle fails at least one of them.
Shapes use dk != dv wherever a transposition could hide.
"""
import numpy as np
import pytest


def unit(rng, *shape):
    x = rng.standard_normal(shape)
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def sig(x):
    return 1.0 / (1.0 + np.exp(-x))


# -------------------------------------------------------------------------
# (1) write hits its target: beta=1, unit k,v => v^T S_t k_t = c_t
#     in general v^T S_t k_t = (1-beta) b_t + c_t  (erase/write split)
# -------------------------------------------------------------------------
@pytest.mark.parametrize("beta_kind", ["one", "general"])
def test_write_hits_target(oracle, beta_kind):
    rng = np.random.default_rng(1)
    dk, dv = 6, 5
    S = rng.standard_normal((dv, dk))
    for t in range(40):
        q, k, v = unit(rng, dk), unit(rng, dk), unit(rng, dv)
        c = rng.standard_normal()
        beta = 1.0 if beta_kind == "one" else 2.0 * sig(rng.standard_normal())
        logf = np.log(sig(rng.normal(2.0, 1.0, dk)))
        Sbar = S * np.exp(logf)[None, :]
        S, o, b, u = oracle.step(S, q, k, v, beta, c, logf)
        assert abs(b - v @ Sbar @ k) < 1e-12
        assoc = v @ S @ k
        assert abs(assoc - ((1.0 - beta) * b + c)) < 1e-12
        if beta_kind == "one":
            assert abs(assoc - c) < 1e-12
        assert np.allclose(o, S @ q, atol=1e-12)


# -------------------------------------------------------------------------
# (2) interference: with f = 1 a stored pair (k_i, v_i) changes by
#     u (v_i . v_t)(k_t . k_i); zero if either key or value is orthogonal
# -------------------------------------------------------------------------
def test_interference_formula_and_orthogonal_protection(oracle):
    rng = np.random.default_rng(2)
    dk, dv = 7, 5
    for trial in range(20):
        S = rng.standard_normal((dv, dk))
        q, k, v = unit(rng, dk), unit(rng, dk), unit(rng, dv)
        beta, c = sig(rng.standard_normal()), rng.standard_normal()
        S1, _, b, u = oracle.step(S, q, k, v, beta, c, np.zeros(dk))
        for _ in range(10):
            ki, vi = unit(rng, dk), unit(rng, dv)
            delta = vi @ S1 @ ki - vi @ S @ ki
            assert abs(delta - u * (vi @ v) * (k @ ki)) < 1e-12
        # key orthogonal to the update key (value arbitrary): untouched
        ki = unit(rng, dk)
        ki = ki - (ki @ k) * k
        ki /= np.linalg.norm(ki)
        vi = unit(rng, dv)
        assert abs(vi @ S1 @ ki - vi @ S @ ki) < 1e-13
        # value orthogonal to the update value (key arbitrary, even equal): untouched
        vi = unit(rng, dv)
        vi = vi - (vi @ v) * v
        vi /= np.linalg.norm(vi)
        for ki in (k, unit(rng, dk)):
            assert abs(vi @ S1 @ ki - vi @ S @ ki) < 1e-13


def test_one_key_holds_orthogonal_values(oracle):
    rng = np.random.default_rng(3)
    dk, dv = 6, 4
    k = unit(rng, dk)
    Vb, _ = np.linalg.qr(rng.standard_normal((dv, dv)))
    S = np.zeros((dv, dk))
    targets = rng.standard_normal(dv)
    for r in range(dv):
        S, *_ = oracle.step(S, k, k, Vb[:, r], 1.0, targets[r], np.zeros(dk))
    for r in range(dv):
        assert abs(Vb[:, r] @ S @ k - targets[r]) < 1e-12


# -------------------------------------------------------------------------
# (3) non-expansive: f <= 1, beta in (0,1) (and (0,2)), unit k,v
# -------------------------------------------------------------------------
@pytest.mark.parametrize("beta_scale", [1.0, 2.0])
def test_non_expansive(oracle, beta_scale):
    rng = np.random.default_rng(4)
    dk, dv = 8, 6
    S, S2 = rng.standard_normal((dv, dk)), rng.standard_normal((dv, dk))
    Z = rng.standard_normal((dv, dk))
    for t in range(100):
        q, k, v = unit(rng, dk), unit(rng, dk), unit(rng, dv)
        beta = beta_scale * sig(rng.standard_normal())
        c = rng.standard_normal()
        logf = np.log(sig(rng.normal(3.0, 1.0, dk)))
        d0 = np.linalg.norm(S - S2)
        S, *_ = oracle.step(S, q, k, v, beta, c, logf)
        S2, *_ = oracle.step(S2, q, k, v, beta, c, logf)
        assert np.linalg.norm(S - S2) <= d0 * (1 + 1e-14) + 1e-15
        n0 = np.linalg.norm(Z)
        Z, *_ = oracle.step(Z, q, k, v, beta, 0.0, logf)
        assert np.linalg.norm(Z) <= n0 * (1 + 1e-14) + 1e-15


# -------------------------------------------------------------------------
# (4) capacity: d_k d_v independent triples stored exactly by sweeps
# -------------------------------------------------------------------------
def test_capacity_kaczmarz(oracle):
    rng = np.random.default_rng(5)
    dk, dv = 4, 4
    n = dk * dv
    while True:
        K, V = unit(rng, n, dk), unit(rng, n, dv)
        Amat = np.stack([np.kron(K[i], V[i]) for i in range(n)])
        if np.linalg.cond(Amat) < 30:
            break
    ctar = rng.standard_normal(n)
    sweeps = 3000
    T = n * sweeps
    idx = np.tile(np.arange(n), sweeps)
    q = np.zeros((1, T, 1, dk))
    k = K[idx][None, :, None, :]
    v = V[idx][None, :, None, :]
    beta = np.ones((1, T, 1))
    c = ctar[idx][None, :, None]
    logf = np.zeros((1, T, 1, dk))
    _, ST = oracle.fwd(q, k, v, beta, c, logf, None, nthreads=1)
    S = ST[0, 0]
    err = max(abs(V[i] @ S @ K[i] - ctar[i]) for i in range(n))
    assert err < 1e-10


# -------------------------------------------------------------------------
# (5) brute force: vectorised form s_t = (I - beta a a^T)(F_t (x) I) s_{t-1} + c a,
#     a = k (x) v, s = vec(S) column-stacked, o_t = (q^T (x) I) s_t
# -------------------------------------------------------------------------
@pytest.mark.parametrize("dk,dv,T", [(4, 3, 12), (3, 4, 9), (2, 2, 7), (4, 4, 5)])
def test_bruteforce_vectorised_products(oracle, dk, dv, T):
    rng = np.random.default_rng(6 + dk * 10 + dv)
    B, H = 1, 2
    q, k, v = unit(rng, B, T, H, dk), unit(rng, B, T, H, dk), unit(rng, B, T, H, dv)
    beta = 2.0 * sig(rng.standard_normal((B, T, H)))
    c = rng.standard_normal((B, T, H))
    logf = np.log(sig(rng.normal(1.0, 1.0, (B, T, H, dk))))
    S0 = rng.standard_normal((B, H, dv, dk))
    O, ST = oracle.fwd(q, k, v, beta, c, logf, S0, nthreads=1)
    n = dk * dv
    I = np.eye(n)
    for h in range(H):
        s0 = S0[0, h].reshape(-1, order="F")
        # explicit products of transition matrices from s_0 to s_t
        Phi = np.eye(n)
        drive = np.zeros(n)
        for t in range(T):
            a = np.kron(k[0, t, h], v[0, t, h])
            Mt = (I - beta[0, t, h] * np.outer(a, a)) @ np.kron(np.diag(np.exp(logf[0, t, h])), np.eye(dv))
            Phi = Mt @ Phi
            drive = Mt @ drive + c[0, t, h] * a
            st = Phi @ s0 + drive
            ot = np.kron(q[0, t, h][None, :], np.eye(dv)) @ st
            assert np.allclose(ot, O[0, t, h], atol=1e-12, rtol=1e-12)
        assert np.allclose(st.reshape(dv, dk, order="F"), ST[0, h], atol=1e-12, rtol=1e-12)


# -------------------------------------------------------------------------
# beta = 0: gated linear attention closed form (no solve)
#   o_t = S0 (gamma_{1:t} . q_t) + sum_{i<=t} c_i v_i (k_i . gamma_{i+1:t})^T q_t
# -------------------------------------------------------------------------
def test_beta_zero_gated_linear_attention(oracle):
    rng = np.random.default_rng(7)
    B, H, T, dk, dv = 1, 2, 40, 5, 3
    q, k, v = unit(rng, B, T, H, dk), unit(rng, B, T, H, dk), unit(rng, B, T, H, dv)
    beta = np.zeros((B, T, H))
    c = rng.standard_normal((B, T, H))
    logf = np.log(sig(rng.normal(1.5, 1.0, (B, T, H, dk))))
    S0 = rng.standard_normal((B, H, dv, dk))
    O, ST = oracle.fwd(q, k, v, beta, c, logf, S0, nthreads=1)
    for h in range(H):
        Lc = np.cumsum(logf[0, :, h], axis=0)  # L_t = sum_{s<=t} logf_s
        for t in range(T):
            o = S0[0, h] @ (np.exp(Lc[t]) * q[0, t, h])
            for i in range(t + 1):
                dec = np.exp(Lc[t] - Lc[i])
                o += c[0, i, h] * v[0, i, h] * ((k[0, i, h] * dec) @ q[0, t, h])
            assert np.allclose(o, O[0, t, h], atol=1e-12)


# -------------------------------------------------------------------------
# d_v = 1, v = 1: the rule is KDA's (per-channel decay delta rule), written
# in the transposed convention S in R^{dk x 1}:
#   S_t = (I - beta k k^T) D_t S_{t-1} + beta k vkda,  vkda = c / beta,
#   o_t = S_t^T q_t
# -------------------------------------------------------------------------
def test_dv1_reduces_to_kda(oracle):
    rng = np.random.default_rng(8)
    B, H, T, dk = 1, 1, 50, 6
    q, k = unit(rng, B, T, H, dk), unit(rng, B, T, H, dk)
    v = np.ones((B, T, H, 1))
    beta = sig(rng.standard_normal((B, T, H))) * 0.9 + 0.05
    c = rng.standard_normal((B, T, H))
    logf = np.log(sig(rng.normal(2.0, 1.0, (B, T, H, dk))))
    O, ST = oracle.fwd(q, k, v, beta, c, logf, None, nthreads=1)
    Sk = np.zeros((dk, 1))
    for t in range(T):
        kt, bt = k[0, t, 0][:, None], beta[0, t, 0]
        Sk = (np.eye(dk) - bt * kt @ kt.T) @ (np.exp(logf[0, t, 0])[:, None] * Sk) + bt * kt * (c[0, t, 0] / bt)
        assert abs((Sk.T @ q[0, t, 0])[0] - O[0, t, 0, 0]) < 1e-12
    assert np.allclose(Sk[:, 0], ST[0, 0, 0], atol=1e-12)


# -------------------------------------------------------------------------
# entry points agree: fwd over T tokens == T decode steps == T single steps
# -------------------------------------------------------------------------
def test_fwd_decode_step_consistency(oracle):
    rng = np.random.default_rng(9)
    B, H, T, dk, dv = 2, 3, 10, 5, 4
    q, k, v = unit(rng, B, T, H, dk), unit(rng, B, T, H, dk), unit(rng, B, T, H, dv)
    beta = sig(rng.standard_normal((B, T, H)))
    c = sig(rng.standard_normal((B, T, H)))
    logf = np.log(sig(rng.normal(3.0, 1.0, (B, T, H, dk))))
    S0 = rng.standard_normal((B, H, dv, dk))
    O, ST, bt, ut = oracle.fwd(q, k, v, beta, c, logf, S0, want_bu=True)
    S = S0.copy()
    for t in range(T):
        S, o = oracle.decode(q[:, t], k[:, t], v[:, t], beta[:, t], c[:, t], logf[:, t], S)
        assert np.array_equal(o, O[:, t])
    assert np.array_equal(S, ST)
    Sx = S0[1, 2].copy()
    for t in range(T):
        Sx, o, b, u = oracle.step(Sx, q[1, t, 2], k[1, t, 2], v[1, t, 2], beta[1, t, 2], c[1, t, 2], logf[1, t, 2])
        assert b == bt[1, t, 2] and u == ut[1, t, 2]
        assert np.array_equal(o, O[1, t, 2])


def test_threads_do_not_change_results(oracle):
    rng = np.random.default_rng(10)
    B, H, T, dk, dv = 2, 3, 70, 6, 5
    q, k, v = unit(rng, B, T, H, dk), unit(rng, B, T, H, dk), unit(rng, B, T, H, dv)
    beta, c = sig(rng.standard_normal((B, T, H))), sig(rng.standard_normal((B, T, H)))
    logf = np.log(sig(rng.normal(3.0, 1.0, (B, T, H, dk))))
    dO = rng.standard_normal((B, T, H, dv))
    a = oracle.fwd(q, k, v, beta, c, logf, None, nthreads=1)
    b = oracle.fwd(q, k, v, beta, c, logf, None, nthreads=4)
    assert all(np.array_equal(x, y) for x, y in zip(a, b))
    g1 = oracle.bwd(q, k, v, beta, c, logf, None, dO, nthreads=1)
    g4 = oracle.bwd(q, k, v, beta, c, logf, None, dO, nthreads=5)
    assert all(np.array_equal(g1[n], g4[n]) for n in g1)


# -------------------------------------------------------------------------
# reverse recurrence vs central finite differences (T = 64, d = 8 slice with
# the state-tracking beta in (0,2); also a T not a multiple of the 64-token
# checkpoint interval)
# -------------------------------------------------------------------------
def _loss(oracle, inp, dO, dST):
    O, ST = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["c"], inp["logf"], inp["S0"], nthreads=1)
    return float(np.sum(O * dO) + np.sum(ST * dST))


@pytest.mark.parametrize("T", [64, 77])
def test_reverse_recurrence_finite_differences(oracle, T):
    rng = np.random.default_rng(11 + T)
    B, H, dk, dv = 1, 2, 8, 8
    inp = dict(q=unit(rng, B, T, H, dk), k=unit(rng, B, T, H, dk), v=unit(rng, B, T, H, dv),
               beta=2.0 * sig(rng.standard_normal((B, T, H))), c=sig(rng.standard_normal((B, T, H))),
               logf=np.exp(rng.uniform(-1, 1)) * np.log(sig(rng.normal(3.0, 1.0, (B, T, H, dk)))),
               S0=rng.standard_normal((B, H, dv, dk)) / 8.0)
    dO = rng.standard_normal((B, T, H, dv))
    dST = rng.standard_normal((B, H, dv, dk))
    g = oracle.bwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["c"], inp["logf"], inp["S0"], dO, dST, nthreads=1)
    names = dict(q="dq", k="dk", v="dv", beta="dbeta", c="dc", logf="dlogf", S0="dS0")
    h = 1e-6
    for name, gname in names.items():
        x0 = inp[name]
        for trial in range(3):  # random unit directions
            d = rng.standard_normal(x0.shape)
            d /= np.linalg.norm(d)
            inp[name] = x0 + h * d
            lp = _loss(oracle, inp, dO, dST)
            inp[name] = x0 - h * d
            lm = _loss(oracle, inp, dO, dST)
            inp[name] = x0
            fd = (lp - lm) / (2 * h)
            an = float(np.sum(g[gname] * d))
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)
        flat = x0.reshape(-1)
        for idx in rng.choice(flat.size, size=min(20, flat.size), replace=False):
            e = np.zeros(flat.size)
            e[idx] = 1.0
            e = e.reshape(x0.shape)
            inp[name] = x0 + h * e
            lp = _loss(oracle, inp, dO, dST)
            inp[name] = x0 - h * e
            lm = _loss(oracle, inp, dO, dST)
            inp[name] = x0
            fd = (lp - lm) / (2 * h)
            an = float(g[gname].reshape(-1)[idx])
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, idx, fd, an)
