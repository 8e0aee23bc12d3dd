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
