"""The Gated DeltaNet-2 chunk form (tests/gdn2_chunk_model.py) equals the
token recurrence of the oracle (oracle/gdn2.py) on ragged lengths, dk != dv
and decays whose in-chunk range is large.  CPU only."""
import numpy as np
import pytest

from oracle import gdn2
from tests import gdn2_chunk_model as cm


@pytest.mark.parametrize("T,dk,dv,C", [(64, 8, 8, 64), (150, 8, 4, 64), (77, 5, 7, 16), (200, 16, 16, 64)])
def test_chunk_form_equals_token_recurrence(T, dk, dv, C):
    r = np.random.default_rng(T + dk)
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)  # noqa: E731
    q, k = unit(r.normal(size=(T, dk))), unit(r.normal(size=(T, dk)))
    v = unit(r.normal(size=(T, dv)))
    b, w = r.uniform(0, 1, size=(T, dk)), r.uniform(0, 1, size=(T, dv))
    loga = -r.uniform(0, 0.3, size=(T, dk))
    S0 = r.normal(size=(dv, dk)) * 0.2
    O, S = gdn2.fwd(*(x[None, :, None] for x in (q, k, v, b, w, loga)), S0[None, None])
    Oc, Sc, _ = cm.chunk_fwd(q, k, v, b, w, loga, S0, C=C)
    assert np.allclose(Oc, O[0, :, 0], rtol=1e-10, atol=1e-12)
    assert np.allclose(Sc, S[0, 0], rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("T,dk,dv,C", [(64, 8, 8, 64), (150, 8, 4, 64), (77, 5, 7, 16)])
def test_chunk_backward_equals_token_backward(T, dk, dv, C):
    r = np.random.default_rng(T * 3 + dv)
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)  # noqa: E731
    q, k = unit(r.normal(size=(T, dk))), unit(r.normal(size=(T, dk)))
    v = unit(r.normal(size=(T, dv)))
    b, w = r.uniform(0, 1, size=(T, dk)), r.uniform(0, 1, size=(T, dv))
    loga = -r.uniform(0, 0.3, size=(T, dk))
    S0 = r.normal(size=(dv, dk)) * 0.2
    dO, dST = r.normal(size=(T, dv)), r.normal(size=(dv, dk))
    g = gdn2.bwd(*(x[None, :, None] for x in (q, k, v, b, w, loga)), S0[None, None], dO[None, :, None],
                 dST[None, None])
    gc = cm.chunk_bwd(q, k, v, b, w, loga, S0, dO, dST, C=C)
    for n in ("dq", "dk", "dv", "db", "dw", "dloga"):
        assert np.allclose(gc[n], g[n][0, :, 0], rtol=1e-9, atol=1e-11), n
    assert np.allclose(gc["dS0"], g["dS0"][0, 0], rtol=1e-9, atol=1e-11)
