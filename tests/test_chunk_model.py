"""The chunk-parallel equations (forward and reverse) agree with the token
oracle; this validates the derivation the CUDA kernels implement."""
import numpy as np
import pytest

from tests.chunk_model import chunk_bwd, chunk_fwd


def unit(rng, *shape):
    x = rng.standard_normal(shape)
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def sig(x):
    return 1.0 / (1.0 + np.exp(-x))


@pytest.mark.parametrize("T,C,dk,dv,beta_scale,s0", [
    (150, 64, 8, 6, 2.0, True), (64, 64, 5, 7, 1.0, False), (37, 16, 6, 6, 2.0, True),
    (1, 64, 4, 4, 1.0, True), (129, 32, 3, 5, 1.0, True)])
def test_chunk_form_matches_oracle(oracle, T, C, dk, dv, beta_scale, s0):
    rng = np.random.default_rng(T * 7 + C)
    B, H = 1, 1
    q, k, v = unit(rng, B, T, H, dk), unit(rng, B, T, H, dk), unit(rng, B, T, H, dv)
    beta = beta_scale * sig(rng.standard_normal((B, T, H)))
    c = sig(rng.standard_normal((B, T, H)))
    logf = 2.0 * np.log(sig(rng.normal(3.0, 1.0, (B, T, H, dk))))
    S0 = rng.standard_normal((B, H, dv, dk)) / 4 if s0 else None
    dO = rng.standard_normal((B, T, H, dv))
    dST = rng.standard_normal((B, H, dv, dk))
    O, ST = oracle.fwd(q, k, v, beta, c, logf, S0)
    g = oracle.bwd(q, k, v, beta, c, logf, S0, dO, dST)
    s0h = None if S0 is None else S0[0, 0]
    Oc, STc, _ = chunk_fwd(q[0, :, 0], k[0, :, 0], v[0, :, 0], beta[0, :, 0], c[0, :, 0], logf[0, :, 0], s0h, C)
    assert np.allclose(Oc, O[0, :, 0], atol=1e-12, rtol=1e-10)
    assert np.allclose(STc, ST[0, 0], atol=1e-12, rtol=1e-10)
    gc = chunk_bwd(q[0, :, 0], k[0, :, 0], v[0, :, 0], beta[0, :, 0], c[0, :, 0], logf[0, :, 0], s0h,
                   dO[0, :, 0], dST[0, 0], C)
    for name, ref in (("dq", g["dq"][0, :, 0]), ("dk", g["dk"][0, :, 0]), ("dv", g["dv"][0, :, 0]),
                      ("dbeta", g["dbeta"][0, :, 0]), ("dc", g["dc"][0, :, 0]),
                      ("dlogf", g["dlogf"][0, :, 0]), ("dS0", g["dS0"][0, 0])):
        assert np.allclose(gc[name], ref, atol=1e-11, rtol=1e-9), name
