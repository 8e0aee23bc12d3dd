"""fp64 CPU oracle for the mixer's input prologue (numpy).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline leg may import this module; the product path never does.  It shares
no code with the CUDA library.

What it computes is the gate and normalisation step that the KronLSTM digest
("KronLSTM이 스칼라 보정으로 긴 문맥 선형 어텐션의 기억 간섭을 줄인다",
section "어떻게 쓰나") places in front of the recurrence, after the layer's
projections, short convolution and SiLU (which stay outside):

  * q, k and v are L2-normalised per token and head;
  * the erase and write gates are sigmoids of their pre-activations, one
    scalar per token and head; for state tracking the erase gate is doubled,
    beta = 2 sigma(.) in (0, 2) (same page, experiments paragraph);
  * the forget gate on key channel j is the sigmoid of its pre-activation
    raised to the head's learned positive exponent a = exp(a_log), so
    log f = exp(a_log) * log sigmoid(x).

Readings (the page gives no formula for them): the L2 normalisation is
x / sqrt(sum x^2 + eps) with eps = 1e-6, and log sigmoid(x) = -softplus(-x).

Shapes: q_raw, k_raw [B,T,H,dk]; v_raw [B,T,H,dv]; beta_pre, c_pre [B,T,H];
f_pre [B,T,H,dk]; a_log [H].  Everything is computed in float64.
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


def log_sigmoid(x):
    """log sigmoid(x) = -softplus(-x), without overflow."""
    x = _f64(x)
    return -(np.maximum(-x, 0.0) + np.log1p(np.exp(-np.abs(x))))


def l2_normalise(x, eps=EPS):
    """Row-wise over the last axis: y = x / sqrt(|x|^2 + eps); also returns 1/sqrt(|x|^2 + eps)."""
    x = _f64(x)
    r = 1.0 / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)
    return x * r, r


def prologue_fwd(q_raw, k_raw, v_raw, beta_pre, c_pre, f_pre, a_log, beta_scale=1.0, eps=EPS):
    """Normalised q, k, v and the gates beta, c, logf the recurrence consumes."""
    q, _ = l2_normalise(q_raw, eps)
    k, _ = l2_normalise(k_raw, eps)
    v, _ = l2_normalise(v_raw, eps)
    beta = beta_scale * sigmoid(beta_pre)
    c = sigmoid(c_pre)
    a = np.exp(_f64(a_log))  # [H]
    logf = a[None, None, :, None] * log_sigmoid(f_pre)
    return dict(q=q, k=k, v=v, beta=beta, c=c, logf=logf)


def prologue_bwd(q_raw, k_raw, v_raw, beta_pre, c_pre, f_pre, a_log, dq, dk, dv, dbeta, dc, dlogf,
                 beta_scale=1.0, eps=EPS):
    """Gradients of the prologue's inputs, given the gradients of its outputs.

    Derived here (the pages ask only for a gate-aware backward):
      y = x r, r = (|x|^2 + eps)^(-1/2)   =>  dx = r (dy - y (y . dy))
      beta = s sigma(b)                    =>  db = dbeta s sigma(b) (1 - sigma(b))
      c = sigma(p)                         =>  dp = dc sigma(p) (1 - sigma(p))
      logf = a log sigma(x), a = e^a_log   =>  dx = dlogf a (1 - sigma(x)),
                                               da_log[h] = sum over (b, t, j) of dlogf logf
    """
    out = {}
    for name, raw, g in (("dq_raw", q_raw, dq), ("dk_raw", k_raw, dk), ("dv_raw", v_raw, dv)):
        y, r = l2_normalise(raw, eps)
        g = _f64(g)
        out[name] = r * (g - y * np.sum(y * g, axis=-1, keepdims=True))
    # 1 - sigmoid(x) is written sigmoid(-x) (the same number, without the
    # cancellation of 1 - sigmoid(x) for large x)
    out["dbeta_pre"] = _f64(dbeta) * beta_scale * sigmoid(beta_pre) * sigmoid(-_f64(beta_pre))
    out["dc_pre"] = _f64(dc) * sigmoid(c_pre) * sigmoid(-_f64(c_pre))
    a = np.exp(_f64(a_log))
    dlogf = _f64(dlogf)
    out["df_pre"] = dlogf * a[None, None, :, None] * sigmoid(-_f64(f_pre))
    logf = a[None, None, :, None] * log_sigmoid(f_pre)
    out["da_log"] = np.sum(dlogf * logf, axis=(0, 1, 3))
    return out
