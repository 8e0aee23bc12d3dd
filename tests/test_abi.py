"""The C ABI library loads, exports every function include/*.h declares, and
rejects bad arguments with the documented error codes before touching the
GPU (no compute calls here; runs without a GPU)."""
import ctypes
import glob
import os
import re

import pytest

import delta_rule_linear_kron_b200 as kd
from delta_rule_linear_kron_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    kbuild.build()
    return kd.lib()


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names |= set(re.findall(r"\b(kron_delta_\w+)\s*\(", src))
    return sorted(names)


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert "kron_delta_fwd" in names and "kron_delta_bwd" in names and "kron_delta_decode" in names
    for n in names:
        assert hasattr(L, n), n


def test_version_and_empty_error(L):
    assert L.kron_delta_version() >= 100
    assert isinstance(L.kron_delta_last_error(), bytes)


def test_workspace_sizes(L):
    B, H, T, d = 1, 16, 16384, 128
    f = kd.workspace_size(kd.KD_WS_FWD, B, H, T, d, d)
    fs = kd.workspace_size(kd.KD_WS_FWD_SAVE, B, H, T, d, d)
    bw = kd.workspace_size(kd.KD_WS_BWD, B, H, T, d, d)
    chunks = B * H * (T // 64)
    assert f >= chunks * (64 + 64 * 64) * 4                      # y, A
    assert fs >= chunks * (64 + 2 * 64 * 64 + d * d + 2 * 64) * 4  # + P, chunk-start states, u, b0
    assert fs >= f
    assert bw >= chunks * (d * d * 2 + 4 * 64 * 64 * 2)  # dS tile and the chunk adjoint tiles (bf16)
    # the fp32 path keeps the chunk-start states only when saving for the backward
    f32 = kd.workspace_size(kd.KD_WS_FWD, B, H, T, d, d, kd.KD_F32)
    assert kd.workspace_size(kd.KD_WS_FWD_SAVE, B, H, T, d, d, kd.KD_F32) >= f32 + chunks * d * d * 4
    # ragged T rounds the chunk count up
    assert kd.workspace_size(kd.KD_WS_FWD, 1, 1, 65, 32, 32) > kd.workspace_size(kd.KD_WS_FWD, 1, 1, 64, 32, 32)
    assert L.kron_delta_workspace_size(0, 1, 1, 64, 48, 32, 1) == 0
    assert b"32, 64 or 128" in L.kron_delta_last_error()
    assert L.kron_delta_workspace_size(12, 1, 1, 64, 32, 32, 1) == 0
    # the backward with recompute holds a save-forward workspace and the backward's
    # own (the CUDA-core path, whose forward always writes an output, one more buffer)
    a256 = lambda x: (x + 255) // 256 * 256  # noqa: E731
    assert kd.workspace_size(kd.KD_WS_BWD_RECOMPUTE, B, H, T, d, d) == a256(fs) + bw
    f32s = kd.workspace_size(kd.KD_WS_FWD_SAVE, B, H, T, d, d, kd.KD_F32)
    f32b = kd.workspace_size(kd.KD_WS_BWD, B, H, T, d, d, kd.KD_F32)
    assert kd.workspace_size(kd.KD_WS_BWD_RECOMPUTE, B, H, T, d, d, kd.KD_F32) == \
        a256(f32s) + a256(B * T * H * d * 4) + f32b


def test_bwd_recompute_rejects_a_short_workspace(L):
    p = ctypes.c_void_p(256)
    need = kd.workspace_size(kd.KD_WS_BWD_RECOMPUTE, 1, 1, 64, 32, 32)
    rc = L.kron_delta_bwd_recompute(p, p, p, p, p, p, None, p, None, p, p, p, p, p, p, None, 1, 1, 64, 32, 32, 1,
                                    p, need - 256, None)
    assert rc == kd.KD_ERR_WORKSPACE
    assert b"recompute" in L.kron_delta_last_error()
    rc = L.kron_delta_bwd_recompute(p, p, p, p, p, None, None, p, None, p, p, p, p, p, p, None, 1, 1, 64, 32, 32, 1,
                                    p, need, None)
    assert rc == kd.KD_ERR_INVALID_ARG and b"logf" in L.kron_delta_last_error()


def _fwd_call(L, **over):
    p = ctypes.c_void_p(256)  # aligned non-null dummy: never dereferenced when validation fails
    args = dict(q=p, k=p, v=p, beta=p, c=p, logf=p, S0=None, out=p, ST=None, B=1, H=1, T=64, dk=32, dv=32,
                dtype=1, ws=p, ws_bytes=0, save=0, stream=None)
    args.update(over)
    return L.kron_delta_fwd(args["q"], args["k"], args["v"], args["beta"], args["c"], args["logf"],
                            args["S0"], args["out"], args["ST"], args["B"], args["H"], args["T"],
                            args["dk"], args["dv"], args["dtype"], args["ws"], args["ws_bytes"],
                            args["save"], args["stream"])


def test_fwd_argument_errors(L):
    assert _fwd_call(L, dk=48) == kd.KD_ERR_UNSUPPORTED
    assert _fwd_call(L, dtype=7) == kd.KD_ERR_UNSUPPORTED
    assert _fwd_call(L, T=0) == kd.KD_ERR_INVALID_ARG
    assert _fwd_call(L, B=-1) == kd.KD_ERR_INVALID_ARG
    assert _fwd_call(L, q=None) == kd.KD_ERR_INVALID_ARG
    assert b"q must not be NULL" in L.kron_delta_last_error()
    assert _fwd_call(L, k=ctypes.c_void_p(258)) == kd.KD_ERR_INVALID_ARG
    assert b"aligned" in L.kron_delta_last_error()
    assert _fwd_call(L, save=2) == kd.KD_ERR_INVALID_ARG
    assert _fwd_call(L, ws_bytes=10) == kd.KD_ERR_WORKSPACE
    need = kd.workspace_size(kd.KD_WS_FWD, 1, 1, 64, 32, 32)
    assert _fwd_call(L, ws_bytes=need, ws=ctypes.c_void_p(256 + 16)) == kd.KD_ERR_WORKSPACE
    assert _fwd_call(L, ws_bytes=need, save=1) == kd.KD_ERR_WORKSPACE


def test_bwd_and_decode_argument_errors(L):
    p = ctypes.c_void_p(256)
    rc = L.kron_delta_bwd(p, p, p, p, p, p, None, p, None, p, p, p, p, p, p, None,
                          1, 1, 64, 32, 32, 1, p, 0, p, 0, None)
    assert rc == kd.KD_ERR_WORKSPACE
    rc = L.kron_delta_bwd(p, p, p, p, p, p, None, None, None, p, p, p, p, p, p, None,
                          1, 1, 64, 32, 32, 1, p, 0, p, 0, None)
    assert rc == kd.KD_ERR_INVALID_ARG
    rc = L.kron_delta_decode(p, p, p, p, p, p, p, p, 1, 1, 128, 96, 1, None)
    assert rc == kd.KD_ERR_UNSUPPORTED
    rc = L.kron_delta_decode(p, p, p, p, p, p, None, p, 1, 1, 128, 128, 1, None)
    assert rc == kd.KD_ERR_INVALID_ARG
    rc = L.kron_delta_decode(p, p, p, p, p, p, p, p, 0, 1, 128, 128, 1, None)
    assert rc == kd.KD_ERR_INVALID_ARG


def test_python_binding_rejects_host_tensors():
    import torch
    q = torch.zeros(1, 64, 1, 32)
    with pytest.raises(kd.KronDeltaError):
        kd.fwd(q, q, q, torch.zeros(1, 64, 1), torch.zeros(1, 64, 1), q)


def _pro_fwd(L, **over):
    p = ctypes.c_void_p(256)
    a = dict(qr=p, kr=p, vr=p, bp=p, cp=p, fp=p, al=p, scale=1.0, q=p, k=p, v=p, beta=p, c=p, logf=p,
             B=1, H=2, T=70, dk=64, dv=32, dtype=1, stream=None)
    a.update(over)
    return L.kron_delta_prologue_fwd(a["qr"], a["kr"], a["vr"], a["bp"], a["cp"], a["fp"], a["al"],
                                     a["scale"], a["q"], a["k"], a["v"], a["beta"], a["c"], a["logf"],
                                     a["B"], a["H"], a["T"], a["dk"], a["dv"], a["dtype"], a["stream"])


def _pro_bwd(L, **over):
    p = ctypes.c_void_p(256)
    a = dict(al=p, scale=2.0, dq=p, dfp=p, da=p, B=1, H=2, T=70, dk=64, dv=32, dtype=1, ws=p, ws_bytes=0)
    a.update(over)
    return L.kron_delta_prologue_bwd(p, p, p, p, p, p, a["al"], a["scale"], a["dq"], p, p, p, p, p,
                                     p, p, p, p, p, a["dfp"], a["da"], a["B"], a["H"], a["T"], a["dk"],
                                     a["dv"], a["dtype"], a["ws"], a["ws_bytes"], None)


def test_prologue_argument_errors(L):
    assert L.kron_delta_prologue_fwd.argtypes[7] is ctypes.c_float
    assert _pro_fwd(L, dk=48) == kd.KD_ERR_UNSUPPORTED
    assert _pro_fwd(L, dtype=3) == kd.KD_ERR_UNSUPPORTED
    assert _pro_fwd(L, T=0) == kd.KD_ERR_INVALID_ARG
    assert _pro_fwd(L, scale=0.0) == kd.KD_ERR_INVALID_ARG
    assert _pro_fwd(L, scale=2.5) == kd.KD_ERR_INVALID_ARG
    assert b"beta_scale" in L.kron_delta_last_error()
    assert _pro_fwd(L, scale=float("nan")) == kd.KD_ERR_INVALID_ARG
    assert _pro_fwd(L, fp=None) == kd.KD_ERR_INVALID_ARG
    assert b"f_pre must not be NULL" in L.kron_delta_last_error()
    assert _pro_fwd(L, logf=ctypes.c_void_p(260)) == kd.KD_ERR_INVALID_ARG
    assert _pro_bwd(L, da=None) == kd.KD_ERR_INVALID_ARG
    assert b"da_log" in L.kron_delta_last_error()
    assert _pro_bwd(L, dq=None) == kd.KD_ERR_INVALID_ARG
    assert _pro_bwd(L) == kd.KD_ERR_WORKSPACE
    need = kd.workspace_size(kd.KD_WS_PROLOGUE_BWD, 1, 2, 70, 64, 32)
    assert need >= 2 * 4 and need % 256 == 0
    assert _pro_bwd(L, ws_bytes=need, ws=ctypes.c_void_p(256 + 64)) == kd.KD_ERR_WORKSPACE
    # one partial per (block of 64 tokens, head)
    big = kd.workspace_size(kd.KD_WS_PROLOGUE_BWD, 2, 16, 16384, 128, 128)
    assert big >= (2 * 16384 // 64) * 16 * 4


def test_epilogue_argument_errors(L):
    p = ctypes.c_void_p(256)
    assert L.kron_delta_epilogue_fwd(p, p, p, p, 1, 2, 10, 96, 1, None) == kd.KD_ERR_UNSUPPORTED
    assert L.kron_delta_epilogue_fwd(p, p, p, p, 1, 2, 10, 64, 5, None) == kd.KD_ERR_UNSUPPORTED
    assert L.kron_delta_epilogue_fwd(p, p, None, p, 1, 2, 10, 64, 1, None) == kd.KD_ERR_INVALID_ARG
    assert b"w must not be NULL" in L.kron_delta_last_error()
    assert L.kron_delta_epilogue_fwd(p, p, p, p, 1, 0, 10, 64, 1, None) == kd.KD_ERR_INVALID_ARG
    assert L.kron_delta_epilogue_bwd(p, p, p, p, p, p, None, 1, 2, 10, 64, 1, p, 1 << 20, None) == \
        kd.KD_ERR_INVALID_ARG
    assert L.kron_delta_epilogue_bwd(p, p, p, p, p, p, p, 1, 2, 10, 64, 1, p, 0, None) == kd.KD_ERR_WORKSPACE
    need = kd.workspace_size(kd.KD_WS_EPILOGUE_BWD, 1, 2, 10, 64, 64)
    assert need >= 64 * 4 and need % 256 == 0
    assert L.kron_delta_epilogue_bwd(p, p, p, p, p, p, p, 1, 2, 10, 64, 1, ctypes.c_void_p(256 + 32), need,
                                     None) == kd.KD_ERR_WORKSPACE
    # partial rows are capped, so the scratch stays small at any size
    assert kd.workspace_size(kd.KD_WS_EPILOGUE_BWD, 64, 64, 65536, 128, 128) <= 4096 * 128 * 4 + 256


def test_phase_argument_errors(L):
    p = ctypes.c_void_p(256)
    for bad in (0, 4, -1):
        rc = L.kron_delta_fwd_phase(p, p, p, p, p, p, None, p, None, 1, 1, 64, 32, 32, 1, p, 1 << 20, 0, bad, None)
        assert rc == kd.KD_ERR_INVALID_ARG
        assert b"phase" in L.kron_delta_last_error()
        rc = L.kron_delta_bwd_phase(p, p, p, p, p, p, None, p, None, p, p, p, p, p, p, None, 1, 1, 64, 32, 32, 1,
                                    p, 1 << 20, p, 1 << 20, bad, None)
        assert rc == kd.KD_ERR_INVALID_ARG
    # a valid phase still validates the rest before touching the GPU
    rc = L.kron_delta_fwd_phase(p, p, p, p, p, p, None, p, None, 1, 1, 64, 48, 32, 1, p, 1 << 20, 0,
                                kd.KD_PHASE_LOCAL, None)
    assert rc == kd.KD_ERR_UNSUPPORTED


def test_gdn2_argument_errors(L):
    p = ctypes.c_void_p(256)
    assert L.kron_delta_gdn2_decode(p, p, p, p, p, p, p, p, 1, 1, 128, 96, 1, None) == kd.KD_ERR_UNSUPPORTED
    assert L.kron_delta_gdn2_decode(p, p, p, p, None, p, p, p, 1, 1, 64, 64, 1, None) == kd.KD_ERR_INVALID_ARG
    assert b"w must not be NULL" in L.kron_delta_last_error()
    assert L.kron_delta_gdn2_fwd(p, p, p, p, p, p, None, p, None, 1, 1, 64, 32, 32, 1, p, 0, None) == \
        kd.KD_ERR_WORKSPACE
    assert L.kron_delta_gdn2_fwd(p, p, p, None, p, p, None, p, None, 1, 1, 64, 32, 32, 1, p, 1 << 30, None) == \
        kd.KD_ERR_INVALID_ARG
    need_f = kd.workspace_size(kd.KD_WS_GDN2_FWD, 1, 2, 100, 64, 32)
    need_b = kd.workspace_size(kd.KD_WS_GDN2_BWD, 1, 2, 100, 64, 32)
    chunks = 2 * 2
    assert need_f >= chunks * (2 * 64 * 64 + 3 * 64 * 64 + 2 * 64 * 32 + 32 * 64) * 4
    assert need_b >= chunks * (64 * 32 + 32 * 64 + 3 * 64 * 64 + 2 * 64 * 64) * 4
    rc = L.kron_delta_gdn2_bwd(p, p, p, p, p, p, None, p, None, p, p, p, p, p, p, None, 1, 2, 100, 64, 32, 1,
                               p, need_f, p, need_b - 256, None)
    assert rc == kd.KD_ERR_WORKSPACE


def test_gdn2_tensor_core_workspace_layout(L):
    """The planner's tensor-core layout for Gated DeltaNet-2 (bf16, d = 128),
    per chunk of C = 64: the forward keeps A, P [C][C], U', Q+, U [C][d] in
    fp32, e^Lambda [d], the chunk-start state as one bf16 image [d][d] and the
    chains' W, K^e images (bf16 hi, lo [C][d]), with no fp32 W, K^e or state;
    the backward adds dU, dE, dQ+, dK^e, P^T dO [C][d], dT, dP [C][C], dS,
    S0 and (dO^T Q+)^T [d][d] in fp32, the dS image in bf16 and one flag byte
    per chunk.  Every region is a multiple of 256 bytes here, so the sizes are
    exact sums."""
    C, d, chunks = 64, 128, 16 * (16384 // 64)
    fwd_floats = 2 * C * C + 3 * C * d + d + d * d // 2 + 2 * C * d
    bwd_floats = 6 * C * d + 2 * C * C + 3 * d * d
    assert kd.workspace_size(kd.KD_WS_GDN2_FWD, 1, 16, 16384, d, d, 1) == chunks * fwd_floats * 4
    assert kd.workspace_size(kd.KD_WS_GDN2_BWD, 1, 16, 16384, d, d, 1) == chunks * bwd_floats * 4 + chunks
    # the CUDA-core layout (fp32 inputs): fp32 W and K^e in place of the two
    # images (the same bytes) and the state in fp32 (twice its bf16 image)
    assert kd.workspace_size(kd.KD_WS_GDN2_FWD, 1, 16, 16384, d, d, 0) == chunks * (fwd_floats + d * d // 2) * 4
