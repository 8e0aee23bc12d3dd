"""Seeded synthetic inputs for the Kronecker delta rule mixer.

This module only draws random inputs; it holds none of the method's
arithmetic.  Both the CUDA path's tests/benchmark and the fp64 oracle consume
what it returns, so the two sides always see bit-identical inputs.

Recipe (shapes and distributions of the five workloads):
  * RNG: numpy PCG64, ``default_rng(seed)``, draws in float64; default seed is
    1000 + workload index.  Draw order: q, k, v, beta-pre, c-pre, a_h,
    logf-pre, S0, dO.
  * q, k, v ~ N(0,1), L2-normalised per token and head in float64, then rounded
    to the storage dtype (bf16 round-to-nearest-even for bf16 workloads).
  * beta = sigmoid(N(0,1)) (times 2 for the state-tracking variant, range
    (0,2)); c = sigmoid(N(0,1)).
  * logf = a_h * log sigmoid(x), x ~ N(3,1) per key channel, a_h = exp(U(-1,1))
    per head (the KronLSTM digest's forget-gate parametrisation f = sigmoid^a).
  * S0: zero, or N(0,1) scaled to Frobenius norm 1 per head.
  * decode states: N(0, 1/128) (variance 1/128).
  * dO ~ N(0,1), rounded to the storage dtype.
  * prologue inputs (``make_prologue_inputs``), drawn in the order q~, k~, v~,
    beta-pre, c-pre, f-pre, a_log, then the upstream gradients dq, dk, dv,
    dbeta, dc, dlogf: raw q~, k~, v~ ~ N(0,1) (storage dtype); beta-pre,
    c-pre ~ N(0,1) (fp32); f-pre ~ N(3,1) (storage dtype); a_log ~ U(-1,1)
    (fp32); upstream gradients N(0,1) (dq, dk, dv in the storage dtype, the
    gate gradients fp32).
  * Gated DeltaNet-2 inputs (``make_gdn2_inputs``), in the order q, k, v, b,
    w, a_h, decay pre-activation, S0, dO: q, k, v as above; erase and write
    gates b = sigmoid(N(0,1)) per key channel, w = sigmoid(N(0,1)) per value
    channel (fp32); loga = -a_h * softplus(x), x ~ N(-4,1), a_h = exp(U(-1,1))
    per head (the article's g = -exp(a) * softplus(.) form, fp32); S0 zero or
    N(0,1) scaled to Frobenius norm 1; dO ~ N(0,1).
  * epilogue inputs (``make_epilogue_inputs``), in the order o, g, w, dy:
    o ~ N(0, 0.1^2) (a read-out's scale), g ~ N(0,1), dy ~ N(0,1) (storage
    dtype); w ~ 1 + N(0, 0.1^2) (fp32).
All arrays are returned as float64 numpy arrays holding exactly the values the
GPU receives (bf16-representable where the dtype is bf16).
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np

__all__ = ["Workload", "WORKLOADS", "make_inputs", "make_gated_inputs", "make_decode_inputs",
           "make_prologue_inputs",
           "make_epilogue_inputs", "make_gdn2_inputs",
           "round_to_dtype", "decode_token_inputs_torch"]


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    dk: int
    dv: int
    dtype: str           # "f32" or "bf16": storage dtype of q, k, v, out, dO
    s0: str              # "zero" or "fro"
    beta_scale: float    # 1.0: beta in (0,1); 2.0: state-tracking, beta in (0,2)
    seed: int


WORKLOADS = {
    1: Workload("tiny-fp32-fwd", 1, 2, 256, 32, 32, "f32", "zero", 1.0, 1001),
    2: Workload("fwd-B4-H16-T2048-d128", 4, 16, 2048, 128, 128, "bf16", "zero", 1.0, 1002),
    3: Workload("fwd-B1-H16-T16384-d128", 1, 16, 16384, 128, 128, "bf16", "fro", 1.0, 1003),
    4: Workload("fwdbwd-B1-H16-T16384-d128-beta2", 1, 16, 16384, 128, 128, "bf16", "fro", 2.0, 1004),
    5: Workload("decode-B256-H16-d128", 256, 16, 1, 128, 128, "bf16", "zero", 1.0, 1005),
}


def round_to_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values to the storage dtype (RNE) and return them as float64."""
    x = np.asarray(x, dtype=np.float64)
    if dtype == "f32":
        return x.astype(np.float32).astype(np.float64)
    if dtype == "bf16":
        f = np.ascontiguousarray(x.astype(np.float32))
        bits = f.view(np.uint32).astype(np.uint64)
        # round-to-nearest-even on the upper 16 bits (inputs are finite)
        rounded = (bits + 0x7FFF + ((bits >> 16) & 1)) & 0xFFFF0000
        return rounded.astype(np.uint32).view(np.float32).astype(np.float64)
    raise ValueError(f"unknown dtype {dtype!r}")


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def _log_sigmoid(x):
    # log sigmoid(x) = -softplus(-x), evaluated without overflow
    return -(np.maximum(-x, 0.0) + np.log1p(np.exp(-np.abs(x))))


def _l2n(x):
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return x / np.maximum(n, 1e-300)


def make_inputs(wl: Workload | int, *, B=None, H=None, T=None, dk=None, dv=None,
                seed=None, beta_scale=None, s0=None, with_dO=True):
    """Draw one workload's inputs.  Shape/seed overrides give smaller parity
    cases with the same distributions.  Returns a dict of float64 arrays:
    q,k [B,T,H,dk], v [B,T,H,dv], beta,c [B,T,H], logf [B,T,H,dk],
    S0 [B,H,dv,dk] or None, dO [B,T,H,dv] (if with_dO), and 'wl'."""
    if isinstance(wl, int):
        wl = WORKLOADS[wl]
    kw = {k_: v_ for k_, v_ in dict(B=B, H=H, T=T, dk=dk, dv=dv, seed=seed,
                                      beta_scale=beta_scale, s0=s0).items() if v_ is not None}
    wl = replace(wl, **kw)
    rng = np.random.default_rng(wl.seed)
    B, H, T, dk, dv = wl.B, wl.H, wl.T, wl.dk, wl.dv
    q = round_to_dtype(_l2n(rng.standard_normal((B, T, H, dk))), wl.dtype)
    k = round_to_dtype(_l2n(rng.standard_normal((B, T, H, dk))), wl.dtype)
    v = round_to_dtype(_l2n(rng.standard_normal((B, T, H, dv))), wl.dtype)
    beta = wl.beta_scale * _sigmoid(rng.standard_normal((B, T, H)))
    c = _sigmoid(rng.standard_normal((B, T, H)))
    a_h = np.exp(rng.uniform(-1.0, 1.0, size=(H,)))
    logf = a_h[None, None, :, None] * _log_sigmoid(rng.normal(3.0, 1.0, size=(B, T, H, dk)))
    # gates are fp32 on the device
    beta = round_to_dtype(beta, "f32")
    c = round_to_dtype(c, "f32")
    logf = round_to_dtype(logf, "f32")
    S0 = None
    if wl.s0 == "fro":
        S0 = rng.standard_normal((B, H, dv, dk))
        S0 = S0 / np.sqrt(np.sum(S0 * S0, axis=(-2, -1), keepdims=True))
        S0 = round_to_dtype(S0, "f32")
    out = dict(q=q, k=k, v=v, beta=beta, c=c, logf=logf, S0=S0, wl=wl)
    if with_dO:
        out["dO"] = round_to_dtype(rng.standard_normal((B, T, H, dv)), wl.dtype)
    return out


def make_gated_inputs(wl: Workload | int, *, seed_gate=3000, **kw):
    """A workload's inputs with the forget gate given as its pre-activation:
    make_inputs(wl, **kw) without logf, plus f_pre [B,T,H,dk] ~ N(3,1) in the
    storage dtype and a_log [H] ~ U(-1,1) (fp32), drawn in that order from
    default_rng(seed_gate) (the prologue inputs' forget-gate distributions)."""
    inp = make_inputs(wl, **kw)
    dtype = (WORKLOADS[wl] if isinstance(wl, int) else wl).dtype
    B, T, H, dk = inp["q"].shape
    rng = np.random.default_rng(seed_gate)
    inp["f_pre"] = round_to_dtype(rng.normal(3.0, 1.0, size=(B, T, H, dk)), dtype)
    inp["a_log"] = round_to_dtype(rng.uniform(-1.0, 1.0, size=(H,)), "f32")
    del inp["logf"]
    return inp


def make_prologue_inputs(B, H, T, dk, dv, dtype="bf16", seed=2000, with_grads=True):
    """Raw inputs of the prologue (and, with_grads, upstream gradients of its
    outputs), as float64 arrays holding the values the GPU receives:
    q_raw, k_raw, f_pre [B,T,H,dk], v_raw [B,T,H,dv], beta_pre, c_pre [B,T,H],
    a_log [H]; dq, dk [B,T,H,dk], dv [B,T,H,dv], dbeta, dc [B,T,H],
    dlogf [B,T,H,dk]."""
    rng = np.random.default_rng(seed)
    out = dict(q_raw=round_to_dtype(rng.standard_normal((B, T, H, dk)), dtype),
               k_raw=round_to_dtype(rng.standard_normal((B, T, H, dk)), dtype),
               v_raw=round_to_dtype(rng.standard_normal((B, T, H, dv)), dtype),
               beta_pre=round_to_dtype(rng.standard_normal((B, T, H)), "f32"),
               c_pre=round_to_dtype(rng.standard_normal((B, T, H)), "f32"),
               f_pre=round_to_dtype(rng.normal(3.0, 1.0, size=(B, T, H, dk)), dtype),
               a_log=round_to_dtype(rng.uniform(-1.0, 1.0, size=(H,)), "f32"))
    if with_grads:
        out.update(dq=round_to_dtype(rng.standard_normal((B, T, H, dk)), dtype),
                   dk=round_to_dtype(rng.standard_normal((B, T, H, dk)), dtype),
                   dv=round_to_dtype(rng.standard_normal((B, T, H, dv)), dtype),
                   dbeta=round_to_dtype(rng.standard_normal((B, T, H)), "f32"),
                   dc=round_to_dtype(rng.standard_normal((B, T, H)), "f32"),
                   dlogf=round_to_dtype(rng.standard_normal((B, T, H, dk)), "f32"))
    return out


def make_gdn2_inputs(B, H, T, dk, dv, dtype="bf16", seed=4000, s0="fro"):
    """Gated DeltaNet-2 inputs as float64 arrays holding the values the GPU
    receives: q, k, b, loga [B,T,H,dk]; v, w, dO [B,T,H,dv]; S0 [B,H,dv,dk] or None."""
    rng = np.random.default_rng(seed)
    q = round_to_dtype(_l2n(rng.standard_normal((B, T, H, dk))), dtype)
    k = round_to_dtype(_l2n(rng.standard_normal((B, T, H, dk))), dtype)
    v = round_to_dtype(_l2n(rng.standard_normal((B, T, H, dv))), dtype)
    b = round_to_dtype(_sigmoid(rng.standard_normal((B, T, H, dk))), "f32")
    w = round_to_dtype(_sigmoid(rng.standard_normal((B, T, H, dv))), "f32")
    a_h = np.exp(rng.uniform(-1.0, 1.0, size=(H,)))
    x = rng.normal(-4.0, 1.0, size=(B, T, H, dk))
    loga = round_to_dtype(-a_h[None, None, :, None] * (np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))), "f32")
    S0 = None
    if s0 == "fro":
        S0 = rng.standard_normal((B, H, dv, dk))
        S0 = round_to_dtype(S0 / np.sqrt(np.sum(S0 * S0, axis=(-2, -1), keepdims=True)), "f32")
    dO = round_to_dtype(rng.standard_normal((B, T, H, dv)), dtype)
    return dict(q=q, k=k, v=v, b=b, w=w, loga=loga, S0=S0, dO=dO)


def make_epilogue_inputs(B, H, T, dv, dtype="bf16", seed=3000):
    """Inputs of the output epilogue as float64 arrays holding the values the GPU
    receives: o, g, dy [B,T,H,dv] and w [dv]."""
    rng = np.random.default_rng(seed)
    return dict(o=round_to_dtype(0.1 * rng.standard_normal((B, T, H, dv)), dtype),
                g=round_to_dtype(rng.standard_normal((B, T, H, dv)), dtype),
                w=round_to_dtype(1.0 + 0.1 * rng.standard_normal(dv), "f32"),
                dy=round_to_dtype(rng.standard_normal((B, T, H, dv)), dtype))


def make_decode_inputs(steps: int, *, B=256, H=16, dk=128, dv=128, dtype="bf16",
                       seed=1005, beta_scale=1.0):
    """Decode workload: state S ~ N(0,1/128) [B,H,dv,dk] and `steps` tokens of
    per-step inputs q,k [steps,B,H,dk], v [steps,B,H,dv], beta,c [steps,B,H],
    logf [steps,B,H,dk]; same distributions as the forward workloads."""
    rng = np.random.default_rng(seed)
    q = round_to_dtype(_l2n(rng.standard_normal((steps, B, H, dk))), dtype)
    k = round_to_dtype(_l2n(rng.standard_normal((steps, B, H, dk))), dtype)
    v = round_to_dtype(_l2n(rng.standard_normal((steps, B, H, dv))), dtype)
    beta = round_to_dtype(beta_scale * _sigmoid(rng.standard_normal((steps, B, H))), "f32")
    c = round_to_dtype(_sigmoid(rng.standard_normal((steps, B, H))), "f32")
    a_h = np.exp(rng.uniform(-1.0, 1.0, size=(H,)))
    logf = round_to_dtype(a_h[None, None, :, None] *
                          _log_sigmoid(rng.normal(3.0, 1.0, size=(steps, B, H, dk))), "f32")
    S = round_to_dtype(rng.normal(0.0, np.sqrt(1.0 / 128.0), size=(B, H, dv, dk)), "f32")
    return dict(q=q, k=k, v=v, beta=beta, c=c, logf=logf, S=S)


def decode_token_inputs_torch(steps: int, *, B=256, H=16, dk=128, dv=128, seed=1005,
                              device="cuda", beta_scale=1.0):
    """Large decode runs (e.g. 1000 steps x 4096 heads) drawn with torch's
    seeded generator directly on the device: same distributions as
    ``make_decode_inputs`` (not the same values).  Returns bf16 q,k,v and fp32
    beta, c, logf, and the fp32 state S."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)

    def unit(shape):
        x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        return (x / x.norm(dim=-1, keepdim=True)).to(torch.bfloat16)

    q = unit((steps, B, H, dk))
    k = unit((steps, B, H, dk))
    v = unit((steps, B, H, dv))
    beta = beta_scale * torch.sigmoid(torch.randn((steps, B, H), generator=g, device=device))
    c = torch.sigmoid(torch.randn((steps, B, H), generator=g, device=device))
    a_h = torch.exp(torch.rand((H,), generator=g, device=device) * 2.0 - 1.0)
    x = torch.randn((steps, B, H, dk), generator=g, device=device) + 3.0
    logf = a_h[None, None, :, None] * torch.nn.functional.logsigmoid(x)
    S = torch.randn((B, H, dv, dk), generator=g, device=device) * (1.0 / 128.0) ** 0.5
    return dict(q=q, k=k, v=v, beta=beta.float(), c=c.float(), logf=logf.float(), S=S.float())
