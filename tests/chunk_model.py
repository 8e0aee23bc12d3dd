"""fp64 numpy model of the chunk-parallel (WY) form of the Kronecker delta rule.

Test infrastructure: it states, in plain numpy, the chunk equations the CUDA
kernels implement, so that the derivation itself is checked against the
token-level oracle before any kernel is trusted.  It is not used by the
product path.

The KronLSTM digest ("KronLSTM이 스칼라 보정으로 긴 문맥 선형 어텐션의 기억
간섭을 줄인다", section "무엇과 다른가") notes that the vectorised rule is a
Widrow-Hoff rule on a_t = k_t (x) v_t with a generalised Householder
transition, so DeltaNet's chunk-parallel training carries over.  Inside one
chunk (positions t = 1..C, state S0 at the chunk start):

  L_t  = sum_{s<=t} logf_s (per key channel),  gamma_t = exp(L_t)
  E_ti = exp(L_t - L_i)  (<= 1 for t >= i)
  M[t,i] = (v_t . v_i) * sum_j k_t[j] k_i[j] E_ti[j]      (i < t)
  P[t,i] = sum_j q_t[j] k_i[j] E_ti[j]                    (i <= t)
  b0_t = v_t^T S0 (k_t * gamma_t)
  u    = (I + diag(beta) M)^{-1} (c - beta * b0)
  O_t  = S0 (q_t * gamma_t) + sum_{i<=t} P[t,i] u_i v_i
  S_C  = S0 diag(gamma_C) + sum_i u_i v_i (k_i * gamma_C / gamma_i)^T

The backward is reverse-mode differentiation of these equations.
"""
import numpy as np


def _chunk_terms(q, k, v, logf):
    L = np.cumsum(logf, axis=0)
    E = np.exp(L[:, None, :] - L[None, :, :])          # [t, i, j]
    n = q.shape[0]
    low = np.tril(np.ones((n, n)), -1)
    lowd = np.tril(np.ones((n, n)), 0)
    GK = np.einsum("tj,ij,tij->ti", k, k, E) * low
    GV = (v @ v.T) * low
    P = np.einsum("tj,ij,tij->ti", q, k, E) * lowd
    return L, E, GK, GV, GK * GV, P


def chunk_fwd(q, k, v, beta, c, logf, S0, C=64):
    """One head.  q,k:[T,dk] v:[T,dv] beta,c:[T] logf:[T,dk] S0:[dv,dk].
    Returns O [T,dv], S_T, and per-chunk saved (S0, u, b, A)."""
    T, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((dv, dk)) if S0 is None else S0.copy()
    O = np.zeros((T, dv))
    saved = []
    for s in range(0, T, C):
        e = min(s + C, T)
        qc, kc, vc, bc, cc, lc = q[s:e], k[s:e], v[s:e], beta[s:e], c[s:e], logf[s:e]
        n = e - s
        L, E, GK, GV, M, P = _chunk_terms(qc, kc, vc, lc)
        gam = np.exp(L)
        Kp, Qp = kc * gam, qc * gam
        Ke = kc * np.exp(L[-1][None, :] - L)
        b0 = np.einsum("tr,rj,tj->t", vc, S, Kp)
        A = np.linalg.inv(np.eye(n) + bc[:, None] * M)
        u = A @ (cc - bc * b0)
        O[s:e] = Qp @ S.T + P @ (u[:, None] * vc)
        saved.append(dict(S0=S.copy(), u=u, b=b0 + M @ u, A=A))
        S = S * gam[-1][None, :] + vc.T @ (u[:, None] * Ke)
    return O, S, saved


def chunk_bwd(q, k, v, beta, c, logf, S0, dO, dST=None, C=64):
    """Reverse-mode of chunk_fwd for one head (loss <dO,O> + <dST,S_T>).
    Returns dict dq, dk, dv, dbeta, dc, dlogf, dS0."""
    T, dk = q.shape
    dv = v.shape[1]
    _, _, saved = chunk_fwd(q, k, v, beta, c, logf, S0, C)
    G = np.zeros((dv, dk)) if dST is None else dST.copy()
    out = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros_like(v),
               dbeta=np.zeros_like(beta), dc=np.zeros_like(c), dlogf=np.zeros_like(logf))
    starts = list(range(0, T, C))
    for ci in reversed(range(len(starts))):
        s = starts[ci]
        e = min(s + C, T)
        n = e - s
        qc, kc, vc, bc, lc, dOc = q[s:e], k[s:e], v[s:e], beta[s:e], logf[s:e], dO[s:e]
        Sv, u, b, A = saved[ci]["S0"], saved[ci]["u"], saved[ci]["b"], saved[ci]["A"]
        L, E, GK, GV, M, P = _chunk_terms(qc, kc, vc, lc)
        gam = np.exp(L)
        gC = gam[-1]
        Kp, Qp = kc * gam, qc * gam
        eC = np.exp(gC[None, :] * 0 + L[-1][None, :] - L)
        Ke = kc * eC
        lowd = np.tril(np.ones((n, n)), 0)
        low = np.tril(np.ones((n, n)), -1)
        dS = G                                            # gradient at the chunk end
        # output and chunk-end read of u
        dOV = dOc @ vc.T                                  # [t, i] = dO_t . v_i
        dP = dOV * u[None, :] * lowd
        du = np.sum(P * dOV, axis=0) + np.einsum("ir,rj,ij->i", vc, dS, Ke)
        g = A.T @ du
        out["dc"][s:e] = g
        out["dbeta"][s:e] = -g * b
        db0 = -bc * g
        dM = -np.outer(bc * g, u) * low
        dGK, dGV = dM * GV, dM * GK
        # state-side products
        dQp = dOc @ Sv                                    # rows: S0^T dO_t
        dKp = db0[:, None] * (vc @ Sv)
        dKe = u[:, None] * (vc @ dS)
        dv_ = (u[:, None] * (P.T @ dOc) + (dGV + dGV.T) @ vc
               + db0[:, None] * (Kp @ Sv.T) + u[:, None] * (Ke @ dS.T))
        # decay-weighted intra-chunk terms (E_ti written out)
        dq_P = np.einsum("ti,ij,tij->tj", dP, kc, E)
        dk_P = np.einsum("ti,tj,tij->ij", dP, qc, E)
        dk_G1 = np.einsum("ti,ij,tij->tj", dGK, kc, E)
        dk_G2 = np.einsum("ti,tj,tij->ij", dGK, kc, E)
        dq_ = dQp * gam + dq_P
        dk_ = dKp * gam + dKe * eC + dk_P + dk_G1 + dk_G2
        dL = (dQp * Qp + dKp * Kp - dKe * Ke + qc * dq_P - kc * dk_P + kc * dk_G1 - kc * dk_G2)
        dL[-1] += np.sum(dKe * Ke, axis=0) + gC * np.sum(dS * Sv, axis=0)
        out["dq"][s:e], out["dk"][s:e], out["dv"][s:e] = dq_, dk_, dv_
        out["dlogf"][s:e] = np.cumsum(dL[::-1], axis=0)[::-1]
        G = dS * gC[None, :] + dOc.T @ Qp + vc.T @ (db0[:, None] * Kp)
    out["dS0"] = G
    return out
