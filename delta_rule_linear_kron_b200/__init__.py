"""Kronecker delta rule (KronLSTM token mixer) for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI of ``libkron_delta.so`` (declared in
``include/kron_delta.h``).  It only marshals arguments: torch provides device
memory and the current stream; every step of the computation runs in the
library's CUDA kernels.  There is no CPU or PyTorch fallback: if the library
is missing, every call raises.

Per head, with fp32 state S (dv x dk), for each token:
    Sbar = S diag(exp(logf)); b = v^T Sbar k; u = c - beta b
    S = Sbar + u v k^T;       o = S q
"""
from __future__ import annotations

import ctypes
import os

__all__ = ["fwd", "bwd", "decode", "fwd_gated", "bwd_gated", "fwd_fused", "bwd_fused",
           "prologue_fwd", "prologue_bwd", "epilogue_fwd", "epilogue_bwd",
           "gdn2_fwd", "gdn2_bwd", "gdn2_decode",
           "workspace_size", "device_status", "library_path",
           "KronDeltaError", "KronDeltaFunction", "PrologueFunction", "EpilogueFunction", "Gdn2Function",
           "KD_WS_FWD", "KD_WS_FWD_SAVE", "KD_WS_BWD"]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libkron_delta.so")
_lib = None

KD_OK, KD_ERR_INVALID_ARG, KD_ERR_UNSUPPORTED, KD_ERR_WORKSPACE, KD_ERR_CUDA, KD_ERR_TIMEOUT = range(6)
KD_F32, KD_BF16 = 0, 1
KD_WS_FWD, KD_WS_FWD_SAVE, KD_WS_BWD, KD_WS_PROLOGUE_BWD, KD_WS_EPILOGUE_BWD = 0, 1, 2, 3, 4
KD_WS_GDN2_FWD, KD_WS_GDN2_BWD = 5, 6
KD_WS_FWD_GATED, KD_WS_BWD_GATED, KD_WS_BWD_RECOMPUTE = 7, 8, 9
KD_WS_FWD_FUSED, KD_WS_BWD_FUSED = 10, 11
KD_PHASE_LOCAL, KD_PHASE_CARRY, KD_PHASE_ALL = 1, 2, 3
_CODES = {1: "KD_ERR_INVALID_ARG", 2: "KD_ERR_UNSUPPORTED", 3: "KD_ERR_WORKSPACE",
          4: "KD_ERR_CUDA", 5: "KD_ERR_TIMEOUT"}


class KronDeltaError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{_CODES.get(code, code)}: {msg}")
        self.code = code


def library_path() -> str:
    return _LIB_PATH


def lib():
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                               "`python -m delta_rule_linear_kron_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        vp, fp, i, sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.kron_delta_version.restype = i
        L.kron_delta_last_error.restype = ctypes.c_char_p
        L.kron_delta_workspace_size.restype = sz
        L.kron_delta_workspace_size.argtypes = [i] * 7
        L.kron_delta_fwd.restype = i
        L.kron_delta_fwd.argtypes = [vp] * 9 + [i] * 6 + [vp, sz, i, vp]
        L.kron_delta_bwd.restype = i
        L.kron_delta_bwd.argtypes = [vp] * 16 + [i] * 6 + [vp, sz, vp, sz, vp]
        L.kron_delta_decode.restype = i
        L.kron_delta_decode.argtypes = [vp] * 8 + [i] * 5 + [vp]
        L.kron_delta_device_status.restype = i
        L.kron_delta_device_status.argtypes = [vp]
        L.kron_delta_fwd_phase.restype = i
        L.kron_delta_fwd_phase.argtypes = [vp] * 9 + [i] * 6 + [vp, sz, i, i, vp]
        L.kron_delta_bwd_phase.restype = i
        L.kron_delta_bwd_phase.argtypes = [vp] * 16 + [i] * 6 + [vp, sz, vp, sz, i, vp]
        L.kron_delta_fwd_noalloc.restype = i
        L.kron_delta_fwd_noalloc.argtypes = [vp] * 9 + [i] * 6 + [vp]
        L.kron_delta_bwd_recompute.restype = i
        L.kron_delta_bwd_recompute.argtypes = [vp] * 16 + [i] * 6 + [vp, sz, vp]
        L.kron_delta_fwd_fused.restype = i
        L.kron_delta_fwd_fused.argtypes = [vp] * 7 + [ctypes.c_float] + [vp] * 3 + [i] * 6 + [vp, sz, i, vp]
        L.kron_delta_bwd_fused.restype = i
        L.kron_delta_bwd_fused.argtypes = [vp] * 7 + [ctypes.c_float] + [vp] * 11 + [i] * 6 + [vp, sz, vp, sz, vp]
        L.kron_delta_fwd_gated.restype = i
        L.kron_delta_fwd_gated.argtypes = [vp] * 10 + [i] * 6 + [vp, sz, i, vp]
        L.kron_delta_bwd_gated.restype = i
        L.kron_delta_bwd_gated.argtypes = [vp] * 18 + [i] * 6 + [vp, sz, vp, sz, vp]
        L.kron_delta_prologue_fwd.restype = i
        L.kron_delta_prologue_fwd.argtypes = [vp] * 7 + [ctypes.c_float] + [vp] * 6 + [i] * 6 + [vp]
        L.kron_delta_prologue_bwd.restype = i
        L.kron_delta_prologue_bwd.argtypes = ([vp] * 7 + [ctypes.c_float] + [vp] * 13 + [i] * 6 +
                                              [vp, sz, vp])
        L.kron_delta_epilogue_fwd.restype = i
        L.kron_delta_epilogue_fwd.argtypes = [vp] * 4 + [i] * 5 + [vp]
        L.kron_delta_epilogue_bwd.restype = i
        L.kron_delta_epilogue_bwd.argtypes = [vp] * 7 + [i] * 5 + [vp, sz, vp]
        L.kron_delta_gdn2_fwd.restype = i
        L.kron_delta_gdn2_fwd.argtypes = [vp] * 9 + [i] * 6 + [vp, sz, vp]
        L.kron_delta_gdn2_bwd.restype = i
        L.kron_delta_gdn2_bwd.argtypes = [vp] * 16 + [i] * 6 + [vp, sz, vp, sz, vp]
        L.kron_delta_gdn2_decode.restype = i
        L.kron_delta_gdn2_decode.argtypes = [vp] * 8 + [i] * 5 + [vp]
        L.kron_delta_selftest_timeout.restype = i
        L.kron_delta_selftest_timeout.argtypes = [vp]
        L.kron_delta_profile_enable.restype = None
        L.kron_delta_profile_enable.argtypes = [i]
        L.kron_delta_profile_report.restype = i
        L.kron_delta_profile_report.argtypes = [ctypes.c_char_p, sz, i]
        _lib = L
    return _lib


def _check(rc):
    if rc != KD_OK:
        raise KronDeltaError(rc, lib().kron_delta_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(t):
    import torch
    if t.dtype == torch.float32:
        return KD_F32
    if t.dtype == torch.bfloat16:
        return KD_BF16
    raise KronDeltaError(KD_ERR_UNSUPPORTED, f"q/k/v dtype {t.dtype} (want float32 or bfloat16)")


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, name, dtype=None, shape=None):
    if t is None:
        return
    if not t.is_cuda:
        raise KronDeltaError(KD_ERR_INVALID_ARG, f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise KronDeltaError(KD_ERR_INVALID_ARG, f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise KronDeltaError(KD_ERR_INVALID_ARG, f"{name} must be {dtype} (got {t.dtype})")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise KronDeltaError(KD_ERR_INVALID_ARG, f"{name} must have shape {tuple(shape)} (got {tuple(t.shape)})")


def workspace_size(kind, B, H, T, dk, dv, dtype=KD_BF16) -> int:
    n = lib().kron_delta_workspace_size(kind, B, H, T, dk, dv, dtype)
    if n == 0:
        raise KronDeltaError(KD_ERR_INVALID_ARG, lib().kron_delta_last_error().decode())
    return n


def _alloc_ws(nbytes, device):
    import torch
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def fwd(q, k, v, beta, c, logf, S0=None, *, out=None, want_state=True, save=False,
        workspace=None, phase=KD_PHASE_ALL, state_out=None, stream=None):
    """Chunk-parallel forward.  q,k [B,T,H,dk], v [B,T,H,dv] (bf16 or fp32);
    beta, c [B,T,H] fp32; logf [B,T,H,dk] fp32; S0 [B,H,dv,dk] fp32 or None.
    Returns (out [B,T,H,dv], ST [B,H,dv,dk] or None, workspace).
    phase: KD_PHASE_LOCAL enqueues only the S0-independent work, KD_PHASE_CARRY
    the rest (pass the LOCAL call's workspace, out and state_out back in)."""
    import torch
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    f32 = torch.float32
    _need(q, "q"); _need(k, "k", q.dtype, q.shape); _need(v, "v", q.dtype, (B, T, H, dv))
    _need(beta, "beta", f32, (B, T, H)); _need(c, "c", f32, (B, T, H))
    _need(logf, "logf", f32, (B, T, H, dk)); _need(S0, "S0", f32, (B, H, dv, dk))
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    _need(out, "out", q.dtype, (B, T, H, dv))
    ST = state_out
    if ST is None and want_state:
        ST = torch.empty((B, H, dv, dk), dtype=f32, device=q.device)
    _need(ST, "state_out", f32, (B, H, dv, dk))
    need = workspace_size(KD_WS_FWD_SAVE if save else KD_WS_FWD, B, H, T, dk, dv, dt)
    if workspace is None:
        workspace = _alloc_ws(need, q.device)
    _check(lib().kron_delta_fwd_phase(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(c), _ptr(logf), _ptr(S0),
                                      _ptr(out), _ptr(ST), B, H, T, dk, dv, dt, _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), int(bool(save)), int(phase),
                                      _stream(stream)))
    return out, ST, workspace


def bwd(q, k, v, beta, c, logf, S0, dO, dST=None, *, fwd_workspace, workspace=None,
        want_dS0=True, phase=KD_PHASE_ALL, grads=None, stream=None):
    """Backward for loss <dO, out> + <dST, ST>, reading what fwd(save=True)
    left in fwd_workspace.  Returns dict dq, dk, dv, dbeta, dc, dlogf, dS0.
    fwd_workspace=None recomputes the forward's chunk quantities instead
    (kron_delta_bwd_recompute; the workspace is then sized by
    KD_WS_BWD_RECOMPUTE and phase must be KD_PHASE_ALL).
    phase: KD_PHASE_LOCAL enqueues only the dST-independent work, KD_PHASE_CARRY
    the rest (allocate the workspace with workspace_size(KD_WS_BWD, ...) and pass
    it, and the LOCAL call's returned grads, to both calls)."""
    import torch
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    f32 = torch.float32
    _need(q, "q"); _need(k, "k", q.dtype, q.shape); _need(v, "v", q.dtype, (B, T, H, dv))
    _need(beta, "beta", f32, (B, T, H)); _need(c, "c", f32, (B, T, H))
    _need(logf, "logf", f32, (B, T, H, dk)); _need(S0, "S0", f32, (B, H, dv, dk))
    _need(dO, "dO", q.dtype, (B, T, H, dv)); _need(dST, "dST", f32, (B, H, dv, dk))
    dt = _dtype_code(q)
    if grads is None:
        g = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
                 dbeta=torch.empty_like(beta), dc=torch.empty_like(c), dlogf=torch.empty_like(logf),
                 dS0=torch.empty((B, H, dv, dk), dtype=f32, device=q.device) if want_dS0 else None)
    else:
        g = grads
        for n, ref in (("dq", q), ("dk", k), ("dv", v), ("dbeta", beta), ("dc", c), ("dlogf", logf)):
            _need(g[n], n, ref.dtype, ref.shape)
        _need(g.get("dS0"), "dS0", f32, (B, H, dv, dk))
    if fwd_workspace is None:
        if phase != KD_PHASE_ALL:
            raise ValueError("recompute (fwd_workspace=None) needs phase=KD_PHASE_ALL")
        if workspace is None:
            workspace = _alloc_ws(workspace_size(KD_WS_BWD_RECOMPUTE, B, H, T, dk, dv, dt), q.device)
        _check(lib().kron_delta_bwd_recompute(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(c), _ptr(logf),
                                              _ptr(S0), _ptr(dO), _ptr(dST), _ptr(g["dq"]), _ptr(g["dk"]),
                                              _ptr(g["dv"]), _ptr(g["dbeta"]), _ptr(g["dc"]), _ptr(g["dlogf"]),
                                              _ptr(g.get("dS0")), B, H, T, dk, dv, dt, _ptr(workspace),
                                              workspace.numel() * workspace.element_size(), _stream(stream)))
        return g
    need = workspace_size(KD_WS_BWD, B, H, T, dk, dv, dt)
    if workspace is None:
        workspace = _alloc_ws(need, q.device)
    _check(lib().kron_delta_bwd_phase(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(c), _ptr(logf), _ptr(S0),
                                      _ptr(dO), _ptr(dST), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]),
                                      _ptr(g["dbeta"]), _ptr(g["dc"]), _ptr(g["dlogf"]), _ptr(g.get("dS0")),
                                      B, H, T, dk, dv, dt, _ptr(fwd_workspace),
                                      fwd_workspace.numel() * fwd_workspace.element_size(),
                                      _ptr(workspace), workspace.numel() * workspace.element_size(), int(phase),
                                      _stream(stream)))
    return g


def fwd_gated(q, k, v, beta, c, f_pre, a_log, S0=None, *, out=None, want_state=True, save=False,
              workspace=None, stream=None):
    """Forward with the forget gate given as its pre-activation: identical to
    fwd on logf = exp(a_log) * log sigmoid(f_pre), with logf formed inside the
    kernels.  f_pre [B,T,H,dk] in q's dtype; a_log [H] fp32.  Returns (out, ST,
    workspace); pass the workspace (save=True) to bwd_gated."""
    import torch
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    f32 = torch.float32
    _need(q, "q"); _need(k, "k", q.dtype, q.shape); _need(v, "v", q.dtype, (B, T, H, dv))
    _need(beta, "beta", f32, (B, T, H)); _need(c, "c", f32, (B, T, H))
    _need(f_pre, "f_pre", q.dtype, (B, T, H, dk)); _need(a_log, "a_log", f32, (H,))
    _need(S0, "S0", f32, (B, H, dv, dk))
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    _need(out, "out", q.dtype, (B, T, H, dv))
    ST = torch.empty((B, H, dv, dk), dtype=f32, device=q.device) if want_state else None
    need = workspace_size(KD_WS_FWD_GATED, B, H, T, dk, dv, dt)
    if workspace is None:
        workspace = _alloc_ws(need, q.device)
    _check(lib().kron_delta_fwd_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(c), _ptr(f_pre), _ptr(a_log),
                                      _ptr(S0), _ptr(out), _ptr(ST), B, H, T, dk, dv, dt, _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), int(bool(save)),
                                      _stream(stream)))
    return out, ST, workspace


def bwd_gated(q, k, v, beta, c, f_pre, a_log, S0, dO, dST=None, *, fwd_workspace, workspace=None,
              want_dS0=True, stream=None):
    """Backward of fwd_gated.  Returns dict dq, dk, dv, dbeta, dc, df_pre
    (fp32), da_log ([H] fp32, summed over the batch in a fixed order), dS0."""
    import torch
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    f32 = torch.float32
    _need(q, "q"); _need(k, "k", q.dtype, q.shape); _need(v, "v", q.dtype, (B, T, H, dv))
    _need(beta, "beta", f32, (B, T, H)); _need(c, "c", f32, (B, T, H))
    _need(f_pre, "f_pre", q.dtype, (B, T, H, dk)); _need(a_log, "a_log", f32, (H,))
    _need(S0, "S0", f32, (B, H, dv, dk))
    _need(dO, "dO", q.dtype, (B, T, H, dv)); _need(dST, "dST", f32, (B, H, dv, dk))
    dt = _dtype_code(q)
    g = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
             dbeta=torch.empty_like(beta), dc=torch.empty_like(c),
             df_pre=torch.empty((B, T, H, dk), dtype=f32, device=q.device),
             da_log=torch.empty((H,), dtype=f32, device=q.device),
             dS0=torch.empty((B, H, dv, dk), dtype=f32, device=q.device) if want_dS0 else None)
    need = workspace_size(KD_WS_BWD_GATED, B, H, T, dk, dv, dt)
    if workspace is None:
        workspace = _alloc_ws(need, q.device)
    _check(lib().kron_delta_bwd_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(c), _ptr(f_pre), _ptr(a_log),
                                      _ptr(S0), _ptr(dO), _ptr(dST), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]),
                                      _ptr(g["dbeta"]), _ptr(g["dc"]), _ptr(g["df_pre"]), _ptr(g["da_log"]),
                                      _ptr(g.get("dS0")), B, H, T, dk, dv, dt, _ptr(fwd_workspace),
                                      fwd_workspace.numel() * fwd_workspace.element_size(),
                                      _ptr(workspace), workspace.numel() * workspace.element_size(),
                                      _stream(stream)))
    return g


def fwd_fused(q_raw, k_raw, v_raw, beta_pre, c_pre, f_pre, a_log, beta_scale, S0=None, *, out=None,
              want_state=True, save=False, workspace=None, stream=None):
    """Forward from the raw projections and gate pre-activations (the input
    prologue fused into the chunk kernels): equal, up to rounding, to
    prologue_fwd followed by fwd.  q_raw, k_raw, f_pre [B,T,H,dk] and v_raw
    [B,T,H,dv] in one dtype; beta_pre, c_pre [B,T,H] and a_log [H] fp32.
    Returns (out, ST, workspace); pass the workspace (save=True) to bwd_fused."""
    import torch
    B, T, H, dk = q_raw.shape
    dv = v_raw.shape[-1]
    f32 = torch.float32
    _need(q_raw, "q_raw"); _need(k_raw, "k_raw", q_raw.dtype, q_raw.shape)
    _need(v_raw, "v_raw", q_raw.dtype, (B, T, H, dv)); _need(f_pre, "f_pre", q_raw.dtype, (B, T, H, dk))
    _need(beta_pre, "beta_pre", f32, (B, T, H)); _need(c_pre, "c_pre", f32, (B, T, H))
    _need(a_log, "a_log", f32, (H,)); _need(S0, "S0", f32, (B, H, dv, dk))
    dt = _dtype_code(q_raw)
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q_raw.dtype, device=q_raw.device)
    _need(out, "out", q_raw.dtype, (B, T, H, dv))
    ST = torch.empty((B, H, dv, dk), dtype=f32, device=q_raw.device) if want_state else None
    if workspace is None:
        workspace = _alloc_ws(workspace_size(KD_WS_FWD_FUSED, B, H, T, dk, dv, dt), q_raw.device)
    _check(lib().kron_delta_fwd_fused(_ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(beta_pre), _ptr(c_pre),
                                      _ptr(f_pre), _ptr(a_log), float(beta_scale), _ptr(S0), _ptr(out), _ptr(ST),
                                      B, H, T, dk, dv, dt, _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), int(bool(save)),
                                      _stream(stream)))
    return out, ST, workspace


def bwd_fused(q_raw, k_raw, v_raw, beta_pre, c_pre, f_pre, a_log, beta_scale, S0, dO, dST=None, *,
              fwd_workspace, workspace=None, want_dS0=True, stream=None):
    """Backward of fwd_fused.  Returns dict dq_raw, dk_raw, dv_raw (input
    dtype), dbeta_pre, dc_pre, df_pre (fp32), da_log ([H] fp32, fixed-order
    sum), dS0."""
    import torch
    B, T, H, dk = q_raw.shape
    dv = v_raw.shape[-1]
    f32 = torch.float32
    _need(q_raw, "q_raw"); _need(k_raw, "k_raw", q_raw.dtype, q_raw.shape)
    _need(v_raw, "v_raw", q_raw.dtype, (B, T, H, dv)); _need(f_pre, "f_pre", q_raw.dtype, (B, T, H, dk))
    _need(beta_pre, "beta_pre", f32, (B, T, H)); _need(c_pre, "c_pre", f32, (B, T, H))
    _need(a_log, "a_log", f32, (H,)); _need(S0, "S0", f32, (B, H, dv, dk))
    _need(dO, "dO", q_raw.dtype, (B, T, H, dv)); _need(dST, "dST", f32, (B, H, dv, dk))
    dt = _dtype_code(q_raw)
    dev = q_raw.device
    g = dict(dq_raw=torch.empty_like(q_raw), dk_raw=torch.empty_like(k_raw), dv_raw=torch.empty_like(v_raw),
             dbeta_pre=torch.empty_like(beta_pre), dc_pre=torch.empty_like(c_pre),
             df_pre=torch.empty((B, T, H, dk), dtype=f32, device=dev),
             da_log=torch.empty((H,), dtype=f32, device=dev),
             dS0=torch.empty((B, H, dv, dk), dtype=f32, device=dev) if want_dS0 else None)
    if workspace is None:
        workspace = _alloc_ws(workspace_size(KD_WS_BWD_FUSED, B, H, T, dk, dv, dt), dev)
    _check(lib().kron_delta_bwd_fused(_ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(beta_pre), _ptr(c_pre),
                                      _ptr(f_pre), _ptr(a_log), float(beta_scale), _ptr(S0), _ptr(dO), _ptr(dST),
                                      _ptr(g["dq_raw"]), _ptr(g["dk_raw"]), _ptr(g["dv_raw"]),
                                      _ptr(g["dbeta_pre"]), _ptr(g["dc_pre"]), _ptr(g["df_pre"]), _ptr(g["da_log"]),
                                      _ptr(g.get("dS0")), B, H, T, dk, dv, dt, _ptr(fwd_workspace),
                                      fwd_workspace.numel() * fwd_workspace.element_size(), _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), _stream(stream)))
    return g


def decode(q, k, v, beta, c, logf, S, *, out=None, stream=None):
    """One decode step.  q,k [B,H,dk], v [B,H,dv], beta,c [B,H], logf [B,H,dk],
    S [B,H,dv,dk] fp32 (updated in place).  Returns out [B,H,dv]."""
    import torch
    B, H, dk = q.shape
    dv = v.shape[-1]
    f32 = torch.float32
    _need(q, "q"); _need(k, "k", q.dtype, q.shape); _need(v, "v", q.dtype, (B, H, dv))
    _need(beta, "beta", f32, (B, H)); _need(c, "c", f32, (B, H)); _need(logf, "logf", f32, (B, H, dk))
    _need(S, "S", f32, (B, H, dv, dk))
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    _need(out, "out", q.dtype, (B, H, dv))
    _check(lib().kron_delta_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(c), _ptr(logf), _ptr(S),
                                   _ptr(out), B, H, dk, dv, dt, _stream(stream)))
    return out


def _prologue_inputs(q_raw, k_raw, v_raw, beta_pre, c_pre, f_pre, a_log):
    import torch
    B, T, H, dk = q_raw.shape
    dv = v_raw.shape[-1]
    f32 = torch.float32
    _need(q_raw, "q_raw"); _need(k_raw, "k_raw", q_raw.dtype, q_raw.shape)
    _need(v_raw, "v_raw", q_raw.dtype, (B, T, H, dv)); _need(f_pre, "f_pre", q_raw.dtype, q_raw.shape)
    _need(beta_pre, "beta_pre", f32, (B, T, H)); _need(c_pre, "c_pre", f32, (B, T, H))
    _need(a_log, "a_log", f32, (H,))
    return B, T, H, dk, dv, _dtype_code(q_raw)


def prologue_fwd(q_raw, k_raw, v_raw, beta_pre, c_pre, f_pre, a_log, beta_scale=1.0, *, stream=None):
    """Input prologue: L2-normalised q, k, v; beta = beta_scale*sigmoid(beta_pre);
    c = sigmoid(c_pre); logf = exp(a_log[h]) * log sigmoid(f_pre).
    q_raw, k_raw, f_pre [B,T,H,dk], v_raw [B,T,H,dv] (bf16 or fp32, one dtype);
    beta_pre, c_pre [B,T,H] fp32; a_log [H] fp32.  Returns dict q, k, v, beta, c, logf
    in the layouts fwd() takes."""
    import torch
    B, T, H, dk, dv, dt = _prologue_inputs(q_raw, k_raw, v_raw, beta_pre, c_pre, f_pre, a_log)
    f32 = torch.float32
    o = dict(q=torch.empty_like(q_raw), k=torch.empty_like(k_raw), v=torch.empty_like(v_raw),
             beta=torch.empty_like(beta_pre), c=torch.empty_like(c_pre),
             logf=torch.empty((B, T, H, dk), dtype=f32, device=q_raw.device))
    _check(lib().kron_delta_prologue_fwd(_ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(beta_pre), _ptr(c_pre),
                                         _ptr(f_pre), _ptr(a_log), float(beta_scale), _ptr(o["q"]),
                                         _ptr(o["k"]), _ptr(o["v"]), _ptr(o["beta"]), _ptr(o["c"]),
                                         _ptr(o["logf"]), B, H, T, dk, dv, dt, _stream(stream)))
    return o


def prologue_bwd(q_raw, k_raw, v_raw, beta_pre, c_pre, f_pre, a_log, dq, dk, dv, dbeta, dc, dlogf,
                 beta_scale=1.0, *, workspace=None, stream=None):
    """Backward of prologue_fwd given the gradients of its outputs (as bwd()
    returns them).  Returns dict dq_raw, dk_raw, dv_raw, dbeta_pre, dc_pre,
    df_pre, da_log."""
    import torch
    B, T, H, dk_, dv_, dt = _prologue_inputs(q_raw, k_raw, v_raw, beta_pre, c_pre, f_pre, a_log)
    f32 = torch.float32
    _need(dq, "dq", q_raw.dtype, (B, T, H, dk_)); _need(dk, "dk", q_raw.dtype, (B, T, H, dk_))
    _need(dv, "dv", q_raw.dtype, (B, T, H, dv_)); _need(dbeta, "dbeta", f32, (B, T, H))
    _need(dc, "dc", f32, (B, T, H)); _need(dlogf, "dlogf", f32, (B, T, H, dk_))
    g = dict(dq_raw=torch.empty_like(q_raw), dk_raw=torch.empty_like(k_raw), dv_raw=torch.empty_like(v_raw),
             dbeta_pre=torch.empty_like(beta_pre), dc_pre=torch.empty_like(c_pre),
             df_pre=torch.empty_like(f_pre), da_log=torch.empty_like(a_log))
    need = workspace_size(KD_WS_PROLOGUE_BWD, B, H, T, dk_, dv_, dt)
    if workspace is None:
        workspace = _alloc_ws(need, q_raw.device)
    _check(lib().kron_delta_prologue_bwd(_ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(beta_pre), _ptr(c_pre),
                                         _ptr(f_pre), _ptr(a_log), float(beta_scale), _ptr(dq), _ptr(dk),
                                         _ptr(dv), _ptr(dbeta), _ptr(dc), _ptr(dlogf), _ptr(g["dq_raw"]),
                                         _ptr(g["dk_raw"]), _ptr(g["dv_raw"]), _ptr(g["dbeta_pre"]),
                                         _ptr(g["dc_pre"]), _ptr(g["df_pre"]), _ptr(g["da_log"]),
                                         B, H, T, dk_, dv_, dt, _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), _stream(stream)))
    return g


def _epilogue_inputs(o, g, w):
    import torch
    B, T, H, dv = o.shape
    _need(o, "o"); _need(g, "g", o.dtype, o.shape); _need(w, "w", torch.float32, (dv,))
    return B, T, H, dv, _dtype_code(o)


def epilogue_fwd(o, g, w, *, out=None, stream=None):
    """Output epilogue: y = w * o / rms(o) * sigmoid(g) per token and head
    (rms over the head's dv channels, eps 1e-6).  o, g [B,T,H,dv] (bf16 or
    fp32, one dtype); w [dv] fp32.  Returns y [B,T,H,dv]."""
    import torch
    B, T, H, dv, dt = _epilogue_inputs(o, g, w)
    y = torch.empty_like(o) if out is None else out
    _need(y, "y", o.dtype, o.shape)
    _check(lib().kron_delta_epilogue_fwd(_ptr(o), _ptr(g), _ptr(w), _ptr(y), B, H, T, dv, dt, _stream(stream)))
    return y


def epilogue_bwd(o, g, w, dy, *, workspace=None, stream=None):
    """Backward of epilogue_fwd for the loss <dy, y>.  Returns dict dO, dg, dw."""
    import torch
    B, T, H, dv, dt = _epilogue_inputs(o, g, w)
    _need(dy, "dy", o.dtype, o.shape)
    r = dict(dO=torch.empty_like(o), dg=torch.empty_like(g), dw=torch.empty_like(w))
    need = workspace_size(KD_WS_EPILOGUE_BWD, B, H, T, 32, dv, dt)
    if workspace is None:
        workspace = _alloc_ws(need, o.device)
    _check(lib().kron_delta_epilogue_bwd(_ptr(o), _ptr(g), _ptr(w), _ptr(dy), _ptr(r["dO"]), _ptr(r["dg"]),
                                         _ptr(r["dw"]), B, H, T, dv, dt, _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), _stream(stream)))
    return r


def _gdn2_inputs(q, k, v, b, w, loga, S0):
    import torch
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    f32 = torch.float32
    _need(q, "q"); _need(k, "k", q.dtype, q.shape); _need(v, "v", q.dtype, (B, T, H, dv))
    _need(b, "b", f32, (B, T, H, dk)); _need(w, "w", f32, (B, T, H, dv)); _need(loga, "loga", f32, (B, T, H, dk))
    _need(S0, "S0", f32, (B, H, dv, dk))
    return B, T, H, dk, dv, _dtype_code(q)


def gdn2_fwd(q, k, v, b, w, loga, S0=None, *, out=None, want_state=True, workspace=None, stream=None):
    """Gated DeltaNet-2 forward: per token Sbar = S diag(exp(loga)),
    u = w*v - Sbar (b*k), S = Sbar + u k^T, o = S q.  q,k [B,T,H,dk], v [B,T,H,dv]
    (bf16 or fp32); b, loga [B,T,H,dk] and w [B,T,H,dv] fp32; S0 [B,H,dv,dk] or
    None.  Returns (out, ST or None, workspace); pass the workspace to gdn2_bwd."""
    import torch
    B, T, H, dk, dv, dt = _gdn2_inputs(q, k, v, b, w, loga, S0)
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    _need(out, "out", q.dtype, (B, T, H, dv))
    ST = torch.empty((B, H, dv, dk), dtype=torch.float32, device=q.device) if want_state else None
    if workspace is None:
        workspace = _alloc_ws(workspace_size(KD_WS_GDN2_FWD, B, H, T, dk, dv, dt), q.device)
    _check(lib().kron_delta_gdn2_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(b), _ptr(w), _ptr(loga), _ptr(S0), _ptr(out),
                                     _ptr(ST), B, H, T, dk, dv, dt, _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream(stream)))
    return out, ST, workspace


def gdn2_bwd(q, k, v, b, w, loga, S0, dO, dST=None, *, fwd_workspace, workspace=None, want_dS0=True,
             stream=None):
    """Backward of gdn2_fwd for the loss <dO, out> + <dST, ST>.  Returns dict
    dq, dk, dv, db, dw, dloga, dS0."""
    import torch
    B, T, H, dk, dv, dt = _gdn2_inputs(q, k, v, b, w, loga, S0)
    f32 = torch.float32
    _need(dO, "dO", q.dtype, (B, T, H, dv)); _need(dST, "dST", f32, (B, H, dv, dk))
    g = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v), db=torch.empty_like(b),
             dw=torch.empty_like(w), dloga=torch.empty_like(loga),
             dS0=torch.empty((B, H, dv, dk), dtype=f32, device=q.device) if want_dS0 else None)
    if workspace is None:
        workspace = _alloc_ws(workspace_size(KD_WS_GDN2_BWD, B, H, T, dk, dv, dt), q.device)
    _check(lib().kron_delta_gdn2_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(b), _ptr(w), _ptr(loga), _ptr(S0), _ptr(dO),
                                     _ptr(dST), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["db"]),
                                     _ptr(g["dw"]), _ptr(g["dloga"]), _ptr(g["dS0"]), B, H, T, dk, dv, dt,
                                     _ptr(fwd_workspace), fwd_workspace.numel() * fwd_workspace.element_size(),
                                     _ptr(workspace), workspace.numel() * workspace.element_size(),
                                     _stream(stream)))
    return g


def gdn2_decode(q, k, v, b, w, loga, S, *, out=None, stream=None):
    """One Gated DeltaNet-2 decode step.  q,k [B,H,dk], v [B,H,dv] (bf16 or fp32);
    b, loga [B,H,dk] and w [B,H,dv] fp32; S [B,H,dv,dk] fp32 (updated in place).
    Returns out [B,H,dv]."""
    import torch
    B, H, dk = q.shape
    dv = v.shape[-1]
    f32 = torch.float32
    _need(q, "q"); _need(k, "k", q.dtype, q.shape); _need(v, "v", q.dtype, (B, H, dv))
    _need(b, "b", f32, (B, H, dk)); _need(w, "w", f32, (B, H, dv)); _need(loga, "loga", f32, (B, H, dk))
    _need(S, "S", f32, (B, H, dv, dk))
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    _need(out, "out", q.dtype, (B, H, dv))
    _check(lib().kron_delta_gdn2_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(b), _ptr(w), _ptr(loga), _ptr(S),
                                        _ptr(out), B, H, dk, dv, dt, _stream(stream)))
    return out


def device_status(stream=None):
    """Synchronise the stream and raise if an earlier call failed on the device."""
    _check(lib().kron_delta_device_status(_stream(stream)))


def _make_function():
    import torch

    class KronDeltaFunction(torch.autograd.Function):
        """autograd wrapper: forward saves what the backward kernels read."""

        @staticmethod
        def forward(ctx, q, k, v, beta, c, logf, S0=None):
            out, ST, ws = fwd(q, k, v, beta, c, logf, S0, save=True)
            ctx.save_for_backward(q, k, v, beta, c, logf, S0, ws)
            return out, ST

        @staticmethod
        def backward(ctx, dO, dST):
            q, k, v, beta, c, logf, S0, ws = ctx.saved_tensors
            g = bwd(q, k, v, beta, c, logf, S0, dO.contiguous(),
                    None if dST is None else dST.contiguous(), fwd_workspace=ws,
                    want_dS0=S0 is not None)
            return g["dq"], g["dk"], g["dv"], g["dbeta"], g["dc"], g["dlogf"], g["dS0"]

    return KronDeltaFunction


def _make_prologue_function():
    import torch

    class PrologueFunction(torch.autograd.Function):
        """autograd wrapper of prologue_fwd / prologue_bwd.  apply(q_raw, k_raw,
        v_raw, beta_pre, c_pre, f_pre, a_log, beta_scale) -> (q, k, v, beta, c, logf)."""

        @staticmethod
        def forward(ctx, q_raw, k_raw, v_raw, beta_pre, c_pre, f_pre, a_log, beta_scale=1.0):
            o = prologue_fwd(q_raw, k_raw, v_raw, beta_pre, c_pre, f_pre, a_log, beta_scale)
            ctx.save_for_backward(q_raw, k_raw, v_raw, beta_pre, c_pre, f_pre, a_log)
            ctx.beta_scale = beta_scale
            return o["q"], o["k"], o["v"], o["beta"], o["c"], o["logf"]

        @staticmethod
        def backward(ctx, dq, dk, dv, dbeta, dc, dlogf):
            saved = ctx.saved_tensors
            z = [torch.zeros_like(t) if g is None else g.contiguous()
                 for g, t in zip((dq, dk, dv, dbeta, dc, dlogf), (saved[0], saved[1], saved[2], saved[3],
                                                                 saved[4], saved[5].float()))]
            g = prologue_bwd(*saved, *z, ctx.beta_scale)
            return g["dq_raw"], g["dk_raw"], g["dv_raw"], g["dbeta_pre"], g["dc_pre"], g["df_pre"], g["da_log"], None

    return PrologueFunction


def _make_epilogue_function():
    import torch

    class EpilogueFunction(torch.autograd.Function):
        """autograd wrapper of epilogue_fwd / epilogue_bwd.  apply(o, g, w) -> y."""

        @staticmethod
        def forward(ctx, o, g, w):
            ctx.save_for_backward(o, g, w)
            return epilogue_fwd(o, g, w)

        @staticmethod
        def backward(ctx, dy):
            o, g, w = ctx.saved_tensors
            r = epilogue_bwd(o, g, w, dy.contiguous())
            return r["dO"], r["dg"], r["dw"]

    return EpilogueFunction


def _make_gdn2_function():
    import torch

    class Gdn2Function(torch.autograd.Function):
        """autograd wrapper of gdn2_fwd / gdn2_bwd.  apply(q, k, v, b, w, loga, S0)
        -> (out, ST)."""

        @staticmethod
        def forward(ctx, q, k, v, b, w, loga, S0=None):
            out, ST, ws = gdn2_fwd(q, k, v, b, w, loga, S0)
            ctx.save_for_backward(q, k, v, b, w, loga, S0, ws)
            return out, ST

        @staticmethod
        def backward(ctx, dO, dST):
            q, k, v, b, w, loga, S0, ws = ctx.saved_tensors
            dO = (torch.zeros((*q.shape[:-1], v.shape[-1]), dtype=q.dtype, device=q.device) if dO is None
                  else dO.contiguous())
            g = gdn2_bwd(q, k, v, b, w, loga, S0, dO, None if dST is None else dST.contiguous(), fwd_workspace=ws,
                         want_dS0=S0 is not None)
            return g["dq"], g["dk"], g["dv"], g["db"], g["dw"], g["dloga"], g["dS0"]

    return Gdn2Function


_LAZY = {"KronDeltaFunction": _make_function, "PrologueFunction": _make_prologue_function,
         "EpilogueFunction": _make_epilogue_function, "Gdn2Function": _make_gdn2_function}


def __getattr__(name):
    if name in _LAZY:
        fn = _LAZY[name]()
        globals()[name] = fn
        return fn
    raise AttributeError(name)
