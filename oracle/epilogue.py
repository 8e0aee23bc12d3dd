"""fp64 CPU oracle for the mixer's output epilogue (numpy).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline leg may import this module; the product path never does.  It shares
no code with the CUDA library.

What it computes: the KronLSTM digest ("KronLSTM이 스칼라 보정으로 긴 문맥 선형
어텐션의 기억 간섭을 줄인다", section "어떻게 쓰나") sends the read-out o_t = S_t q_t
through a sigmoid output gate and a per-head RMSNorm before the output
projection (which stays outside).

Readings (the page names the two operations but gives neither formula nor
order): the norm comes first and the gate multiplies its result,

    y = w * o / sqrt(mean_j(o_j^2) + eps) * sigmoid(g),     eps = 1e-6,

per token and head, the mean over the head's dv channels, w [dv] a learned
per-channel weight shared by the heads, g the gate's pre-activation [dv] per
token and head.

Shapes: o, g [B,T,H,dv]; w [dv].  Everything is computed in float64.
"""
from __future__ import annotations

import numpy as np

EPS = 1e-6


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def sigmoid(x):
    x = _f64(x)
    out = np.empty_like(x)
    pos = x >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-x[pos]))
    ex = np.exp(x[~pos])
    out[~pos] = ex / (1.0 + ex)
    return out


def rms_normalise(o, eps=EPS):
    """o / sqrt(mean(o^2) + eps) over the last axis; also returns the reciprocal RMS."""
    o = _f64(o)
    r = 1.0 / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps)
    return o * r, r


def epilogue_fwd(o, g, w, eps=EPS):
    n, _ = rms_normalise(o, eps)
    return _f64(w) * n * sigmoid(g)


def epilogue_bwd(o, g, w, dy, eps=EPS):
    """Gradients of o, g and w for the loss <dy, y>.

    Derived here:
      n = o r, r = (mean o^2 + eps)^(-1/2), s = sigmoid(g), y = w n s
      dn = dy w s;  do = r (dn - n mean(n dn))
      dg = dy w n s (1 - s) = dy w n sigmoid(g) sigmoid(-g)
      dw = sum over tokens and heads of dy n s
    """
    n, r = rms_normalise(o, eps)
    w = _f64(w)
    dy = _f64(dy)
    g = _f64(g)
    s = sigmoid(g)
    dn = dy * w * s
    do = r * (dn - n * np.mean(n * dn, axis=-1, keepdims=True))
    dg = dy * w * n * s * sigmoid(-g)
    dw = np.sum(dy * n * s, axis=tuple(range(o.ndim - 1)))
    return dict(do=do, dg=dg, dw=dw)
