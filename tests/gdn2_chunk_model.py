"""fp64 numpy model of the chunk-parallel (WY) form of the Gated DeltaNet-2
recurrence, in the library's state convention (S in R^{dv x dk}, o = S q).

Test infrastructure: it states the chunk equations the CUDA kernels implement
so that the derivation is checked against the token oracle (oracle/gdn2.py)
before any kernel is trusted.  Gated DeltaNet-2 article, section "방법론",
step 3: with the decay absorbed, E = gamma o (B o K), Z = W o V,
T = tril(E K^T, -1) (keys divided by their decay), A = (I + T)^{-1},
U = A Z, Y = A E.  Inside one chunk (state S0 at its start):

  L_t = sum_{s<=t} loga_s,  gamma_t = exp(L_t),  Lambda = L at the chunk end
  E+_t = (b_t o k_t) o gamma_t,   K-_i = k_i / gamma_i,   Q+_t = q_t o gamma_t
  T[t,i] = E+_t . K-_i  (i < t),  P[t,i] = Q+_t . K-_i  (i <= t)
  A = (I + T)^{-1},  W = A E+,  U' = A (w o v)
  U = U' - W S0^T                           (row t: u_t = z_t - Sbar_t e_t)
  O = Q+ S0^T + P U
  S_C = S0 diag(exp(Lambda)) + U^T K^e,     K^e_i = k_i o exp(Lambda - L_i)
"""
import numpy as np


def chunk_fwd(q, k, v, b, w, loga, S0, C=64):
    """One head.  q, k, b, loga: [T, dk]; v, w: [T, dv]; S0: [dv, dk] or None.
    Returns O [T, dv], S_T and the chunk-start states."""
    T, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((dv, dk)) if S0 is None else S0.copy()
    O = np.zeros((T, dv))
    starts = []
    for s in range(0, T, C):
        e = min(s + C, T)
        n = e - s
        L = np.cumsum(loga[s:e], axis=0)
        gam = np.exp(L)
        Ep = b[s:e] * k[s:e] * gam
        Km = k[s:e] / gam
        Qp = q[s:e] * gam
        Ke = k[s:e] * np.exp(L[-1][None, :] - L)
        Tm = np.tril(Ep @ Km.T, -1)
        P = np.tril(Qp @ Km.T, 0)
        A = np.linalg.inv(np.eye(n) + Tm)
        W = A @ Ep
        Up = A @ (w[s:e] * v[s:e])
        starts.append(S.copy())
        U = Up - W @ S.T
        O[s:e] = Qp @ S.T + P @ U
        S = S * np.exp(L[-1])[None, :] + U.T @ Ke
    return O, S, starts
