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


def chunk_bwd(q, k, v, b, w, loga, S0, dO, dST=None, C=64):
    """Reverse-mode of chunk_fwd, chunk by chunk, in the form the CUDA kernels
    use (the decay weights exp(L_t - L_i) taken per element).  Returns dict
    dq, dk, dv, db, dw, dloga, dS0.

    Per chunk, given dS (gradient of the chunk-end state):
      dU   = P^T dO + K^e dS^T                       (reverse chain, with
      dS0  = dO^T Q+ + dS Gamma - dU^T W              the next line)
      dP   = tril(dO U^T);  dQ+ = dO S0;  dK^e = U dS;  dW = -dU S0
      dZ   = A^T dU;  dE = A^T dW;  dT = -tril(dZ U'^T + dE W^T, -1)
      then through E+ = e o gamma, Q+ = q o gamma, K^e = k o exp(Lambda - L),
      T, P (exact weights), e = b o k, Z = w o v, and L = cumsum(loga).
    """
    T, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((dv, dk)) if S0 is None else S0.copy()
    chunks = []
    for s in range(0, T, C):
        e_ = min(s + C, T)
        n = e_ - s
        L = np.cumsum(loga[s:e_], axis=0)
        gam = np.exp(L)
        ee = b[s:e_] * k[s:e_]
        Ep, Qp = ee * gam, q[s:e_] * gam
        Ke = k[s:e_] * np.exp(L[-1][None, :] - L)
        Wt = np.exp(L[:, None, :] - L[None, :, :])           # [t, i, j]
        Tm = np.tril(np.einsum("tj,ij,tij->ti", ee, k[s:e_], Wt), -1)
        P = np.tril(np.einsum("tj,ij,tij->ti", q[s:e_], k[s:e_], Wt), 0)
        A = np.linalg.inv(np.eye(n) + Tm)
        W = A @ Ep
        Z = w[s:e_] * v[s:e_]
        Up = A @ Z
        U = Up - W @ S.T
        chunks.append(dict(s=s, e=e_, L=L, gam=gam, ee=ee, Ep=Ep, Qp=Qp, Ke=Ke, Wt=Wt, P=P, A=A, W=W, Z=Z, Up=Up,
                           U=U, S0=S.copy()))
        S = S * np.exp(L[-1])[None, :] + U.T @ Ke
    out = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros_like(v), db=np.zeros_like(b),
               dw=np.zeros_like(w), dloga=np.zeros_like(loga))
    dS = np.zeros((dv, dk)) if dST is None else dST.copy()
    for ch in reversed(chunks):
        s, e_ = ch["s"], ch["e"]
        dOc = dO[s:e_]
        gC = np.exp(ch["L"][-1])
        dU = ch["P"].T @ dOc + ch["Ke"] @ dS.T
        dS_prev = dOc.T @ ch["Qp"] + dS * gC[None, :] - dU.T @ ch["W"]
        # chunk-local gradients
        dP = np.tril(dOc @ ch["U"].T, 0)
        dQp = dOc @ ch["S0"]
        dKe = ch["U"] @ dS
        dW = -dU @ ch["S0"]
        dZ = ch["A"].T @ dU
        dE = ch["A"].T @ dW
        dT = -np.tril(dZ @ ch["Up"].T + dE @ ch["W"].T, -1)
        gam, L, ee, kc, qc = ch["gam"], ch["L"], ch["ee"], k[s:e_], q[s:e_]
        dee = dE * gam
        dL = dE * ch["Ep"] + dQp * ch["Qp"] - dKe * ch["Ke"]
        dqc = dQp * gam
        dkc = dKe * np.exp(L[-1][None, :] - L)
        # exact-weight terms of T and P
        Wt = ch["Wt"]
        dee += np.einsum("ti,ij,tij->tj", dT, kc, Wt)
        dqc += np.einsum("ti,ij,tij->tj", dP, kc, Wt)
        side = dT[:, :, None] * ee[:, None, :] + dP[:, :, None] * qc[:, None, :]   # [t, i, j]
        dkc += np.einsum("tij,tij->ij", side, Wt)
        contrib = side * kc[None, :, :] * Wt                                     # d/dL_t (+), d/dL_i (-)
        dL += contrib.sum(axis=1) - contrib.sum(axis=0)
        dLam = np.sum(dS * ch["S0"], axis=0) * gC + np.sum(dKe * ch["Ke"], axis=0)
        out["dq"][s:e_] = dqc
        out["dk"][s:e_] = dkc + dee * b[s:e_]
        out["db"][s:e_] = dee * kc
        out["dv"][s:e_] = dZ * w[s:e_]
        out["dw"][s:e_] = dZ * v[s:e_]
        out["dloga"][s:e_] = np.cumsum(dL[::-1], axis=0)[::-1] + dLam[None, :]
        dS = dS_prev
    out["dS0"] = dS
    return out
