"""fp64 CPU oracle for the Gated DeltaNet-2 token recurrence (numpy).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline leg may import this module; the product path never does.  It shares
no code with the CUDA library.

Gated DeltaNet-2 article (aitrends.kr), sections "핵심 기여" and "방법론":
the erase gate b_t (one value per key channel) and the write gate w_t (one
per value channel) are decoupled, e_t = b_t o k_t, z_t = w_t o v_t, and with
the channel-wise decay absorbed first,

    S_t = (I - k_t e_t^T) D_t S_{t-1} + k_t z_t^T,   o_t = S_t^T q_t

in the article's convention (S in R^{dk x dv}).  This module keeps the
KronLSTM convention used by the rest of the library (S in R^{dv x dk}, decay
from the right, o = S q), i.e. the transpose of the article's state:

    Sbar_t = S_{t-1} diag(exp(loga_t))
    u_t    = z_t - Sbar_t e_t                 (dv)
    S_t    = Sbar_t + u_t k_t^T
    o_t    = S_t q_t

loga_t [dk] is the log of the channel decay (<= 0).  Shapes: q, k, b, loga
[B,T,H,dk]; v, w [B,T,H,dv]; S0 [B,H,dv,dk] or None.  The time loop is plain
Python over tokens, vectorised over (B, H) only.
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    return None if x is None else np.asarray(x, dtype=np.float64)


def fwd(q, k, v, b, w, loga, S0=None):
    """Returns (O [B,T,H,dv], S_T [B,H,dv,dk])."""
    q, k, v, b, w, loga, S0 = map(_f64, (q, k, v, b, w, loga, S0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    S = np.zeros((B, H, dv, dk)) if S0 is None else S0.copy()
    O = np.zeros((B, T, H, dv))
    for t in range(T):
        Sbar = S * np.exp(loga[:, t])[:, :, None, :]
        e = b[:, t] * k[:, t]
        u = w[:, t] * v[:, t] - np.einsum("bhrj,bhj->bhr", Sbar, e)
        S = Sbar + u[..., :, None] * k[:, t][..., None, :]
        O[:, t] = np.einsum("bhrj,bhj->bhr", S, q[:, t])
    return O, S


def bwd(q, k, v, b, w, loga, S0, dO, dST=None):
    """Reverse-mode recurrence for the loss <dO, O> + <dST, S_T>.
    Returns dict dq, dk, dv, db, dw, dloga, dS0.

    Derived here (the article asks for a gate-aware backward).  With G the
    gradient of S_t and the forward step Sbar = S_{t-1} D, u = z - Sbar e,
    S_t = Sbar + u k^T, o = S_t q:
      G += dO_t q^T;          dq = S_t^T dO_t
      du = G k;               dk  = G^T u            (from the write)
      dz = du;                dSbar = G - du e^T;    de = -Sbar^T du
      db = de o k;            dk += de o b;          dw = dz o v;   dv = dz o w
      dloga_j = sum_r dSbar[r,j] Sbar[r,j];          G_{t-1} = dSbar D
    The states are recomputed by a forward pass kept in memory (small cases).
    """
    q, k, v, b, w, loga, S0, dO, dST = map(_f64, (q, k, v, b, w, loga, S0, dO, dST))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    S = np.zeros((B, H, dv, dk)) if S0 is None else S0.copy()
    states = [S]
    for t in range(T):
        Sbar = S * np.exp(loga[:, t])[:, :, None, :]
        e = b[:, t] * k[:, t]
        u = w[:, t] * v[:, t] - np.einsum("bhrj,bhj->bhr", Sbar, e)
        S = Sbar + u[..., :, None] * k[:, t][..., None, :]
        states.append(S)
    G = np.zeros((B, H, dv, dk)) if dST is None else dST.copy()
    out = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros_like(v), db=np.zeros_like(b),
               dw=np.zeros_like(w), dloga=np.zeros_like(loga))
    for t in reversed(range(T)):
        Sprev, St = states[t], states[t + 1]
        D = np.exp(loga[:, t])
        Sbar = Sprev * D[:, :, None, :]
        kt, qt, bt, wt, vt = k[:, t], q[:, t], b[:, t], w[:, t], v[:, t]
        e = bt * kt
        u = wt * vt - np.einsum("bhrj,bhj->bhr", Sbar, e)
        G = G + dO[:, t][..., :, None] * qt[..., None, :]
        out["dq"][:, t] = np.einsum("bhrj,bhr->bhj", St, dO[:, t])
        du = np.einsum("bhrj,bhj->bhr", G, kt)
        dk_t = np.einsum("bhrj,bhr->bhj", G, u)
        dSbar = G - du[..., :, None] * e[..., None, :]
        de = -np.einsum("bhrj,bhr->bhj", Sbar, du)
        out["db"][:, t] = de * kt
        out["dk"][:, t] = dk_t + de * bt
        out["dw"][:, t] = du * vt
        out["dv"][:, t] = du * wt
        out["dloga"][:, t] = np.einsum("bhrj,bhrj->bhj", dSbar, Sbar)
        G = dSbar * D[:, :, None, :]
    out["dS0"] = G
    return out
