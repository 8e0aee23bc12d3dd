"""fp64 CPU oracle for the Kronecker delta rule token mixer (ctypes binding).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline leg may import this module; the product path never does.  It loads
``libkd_oracle.so`` built from ``kd_oracle.c`` in this directory (see
``build_oracle``), which shares no code with the CUDA library.

What it computes is the token recurrence of the KronLSTM digest ("KronLSTM이
스칼라 보정으로 긴 문맥 선형 어텐션의 기억 간섭을 줄인다", sections "어떻게
동작하나" and "어떻게 쓰나"), in double precision, one token after another:

    Sbar = S diag(exp(logf));  b = v^T Sbar k;  u = c - beta b
    S = Sbar + u v k^T;        o = S q

and its reverse-mode recurrence.  Every array handed in is converted to
float64 (bf16 inputs are upcast exactly).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kd_oracle.c")
_LIB = os.path.join(_HERE, "libkd_oracle.so")
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)


def build_oracle(force: bool = False) -> str:
    """Compile kd_oracle.c with gcc (-O2, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
               "-fPIC", "-shared", "-pthread", "-D_POSIX_C_SOURCE=200809L",
               _SRC, "-o", _LIB, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build_oracle()
        lib = ctypes.CDLL(_LIB)
        i, d = ctypes.c_int, ctypes.c_double
        lib.kdo_step.argtypes = [_dp, _dp, _dp, _dp, d, d, _dp, i, i, _dp, _dp, _dp]
        lib.kdo_fwd.argtypes = [_dp] * 11 + [i] * 6
        lib.kdo_bwd.argtypes = [_dp] * 16 + [i] * 6
        lib.kdo_decode.argtypes = [_dp] * 8 + [i] * 4
        for f in (lib.kdo_step, lib.kdo_fwd, lib.kdo_bwd, lib.kdo_decode):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: exact upcast on the host
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


def step(S, q, k, v, beta, c, logf):
    """One token for one head.  Returns (S_new, o, b, u); S is not modified."""
    lib = _load()
    S = _f64(S).copy()
    q, k, v, logf = _f64(q), _f64(k), _f64(v), _f64(logf)
    dv, dk = S.shape
    o = np.zeros(dv)
    b = ctypes.c_double()
    u = ctypes.c_double()
    rc = lib.kdo_step(_ptr(S), _ptr(q), _ptr(k), _ptr(v), float(beta), float(c),
                      _ptr(logf), dk, dv, _ptr(o), ctypes.byref(b), ctypes.byref(u))
    if rc:
        raise RuntimeError("kdo_step failed")
    return S, o, b.value, u.value


def fwd(q, k, v, beta, c, logf, S0=None, nthreads=0, want_bu=False):
    """Token recurrence for all (b,h).  q,k:[B,T,H,dk] v:[B,T,H,dv] beta,c:[B,T,H]
    logf:[B,T,H,dk] S0:[B,H,dv,dk] or None.  Returns (O, ST) or (O, ST, b, u)."""
    lib = _load()
    q, k, v, beta, c, logf, S0 = map(_f64, (q, k, v, beta, c, logf, S0))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    O = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dv, dk))
    bt = np.zeros((B, T, H)) if want_bu else None
    ut = np.zeros((B, T, H)) if want_bu else None
    rc = lib.kdo_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(c), _ptr(logf),
                     _ptr(S0), _ptr(O), _ptr(ST), _ptr(bt), _ptr(ut),
                     B, H, T, dk, dv, int(nthreads))
    if rc:
        raise RuntimeError("kdo_fwd failed")
    return (O, ST, bt, ut) if want_bu else (O, ST)


def bwd(q, k, v, beta, c, logf, S0, dO, dST=None, nthreads=0):
    """Reverse-mode recurrence.  Returns dict dq, dk, dv, dbeta, dc, dlogf, dS0."""
    lib = _load()
    q, k, v, beta, c, logf, S0, dO, dST = map(_f64, (q, k, v, beta, c, logf, S0, dO, dST))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    out = dict(dq=np.zeros_like(q), dk=np.zeros_like(k), dv=np.zeros_like(v),
               dbeta=np.zeros_like(beta), dc=np.zeros_like(c),
               dlogf=np.zeros_like(logf), dS0=np.zeros((B, H, dv, dk)))
    rc = lib.kdo_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(c), _ptr(logf),
                     _ptr(S0), _ptr(dO), _ptr(dST), _ptr(out["dq"]), _ptr(out["dk"]),
                     _ptr(out["dv"]), _ptr(out["dbeta"]), _ptr(out["dc"]),
                     _ptr(out["dlogf"]), _ptr(out["dS0"]), B, H, T, dk, dv, int(nthreads))
    if rc:
        raise RuntimeError("kdo_bwd failed")
    return out


def decode(q, k, v, beta, c, logf, S):
    """One token per (b,h).  Returns (S_new, o); the input S is not modified."""
    lib = _load()
    q, k, v, beta, c, logf = map(_f64, (q, k, v, beta, c, logf))
    S = _f64(S).copy()
    B, H, dv, dk = S.shape
    o = np.zeros((B, H, dv))
    rc = lib.kdo_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(c), _ptr(logf),
                        _ptr(S), _ptr(o), B, H, dk, dv)
    if rc:
        raise RuntimeError("kdo_decode failed")
    return S, o
