"""kron_delta_fwd_noalloc: the forward for callers that cannot allocate device
memory at call time (for instance a process whose device memory is all
reserved by another allocator).  Its scratch is a fixed 32 MiB array inside
the library, so it must give the same results as kron_delta_fwd with a
caller-provided workspace, call after call, even though the array keeps the
previous call's contents.

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest

import delta_rule_linear_kron_b200 as kd
from delta_rule_linear_kron_b200 import inputs as kin

TOL_BF16 = 5e-3  # the bf16 forward tolerance used by the parity tests


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def test_rejects_problems_beyond_the_fixed_scratch():
    L = kd.lib()
    p = ctypes.c_void_p(256)  # never dereferenced: the call is rejected first
    # the largest bf16 d = 128 problem (in chunk-heads B*H*ceil(T/64)) per the library's own planner
    n = 1
    while kd.workspace_size(kd.KD_WS_FWD, 1, 1, (n + 1) * 64, 128, 128) <= 32 << 20:
        n += 1
    assert n >= 144  # the GPU case below uses 144
    rc = L.kron_delta_fwd_noalloc(p, p, p, p, p, p, None, p, None, 1, 1, (n + 1) * 64, 128, 128, 1, None)
    assert rc == kd.KD_ERR_WORKSPACE
    assert b"exceeds the fixed" in L.kron_delta_last_error()
    # fp32 (CUDA-core path): 1016 chunk-heads fit, 1017 do not
    assert kd.workspace_size(kd.KD_WS_FWD, 1, 1, 1016 * 64, 128, 128, kd.KD_F32) <= 32 << 20
    rc = L.kron_delta_fwd_noalloc(p, p, p, p, p, p, None, p, None, 1, 1, 1017 * 64, 128, 128, 0, None)
    assert rc == kd.KD_ERR_WORKSPACE
    rc = L.kron_delta_fwd_noalloc(p, p, p, p, p, p, None, p, None, 1, 1, 64, 96, 128, 1, None)
    assert rc == kd.KD_ERR_UNSUPPORTED


def _noalloc(L, d, dtype_code):
    import torch
    B, T, H, dk = d["q"].shape
    dv = d["v"].shape[-1]
    out = torch.full((B, T, H, dv), float("nan"), dtype=d["q"].dtype, device="cuda")
    ST = torch.full((B, H, dv, dk), float("nan"), dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = L.kron_delta_fwd_noalloc(_p(d["q"]), _p(d["k"]), _p(d["v"]), _p(d["beta"]), _p(d["c"]),
                                  _p(d["logf"]), _p(d.get("S0")), _p(out), _p(ST), B, H, T, dk, dv,
                                  dtype_code, stream)
    assert rc == kd.KD_OK, L.kron_delta_last_error()
    torch.cuda.synchronize()
    return out, ST


@pytest.mark.gpu
def test_noalloc_matches_workspace_forward_twice(oracle):
    """Larger problem first, then smaller ones, so later calls run on the
    array's leftover contents; each result must equal the workspace forward
    bit for bit (the forward is deterministic), and one is also held against
    the fp64 oracle."""
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU test needs a CUDA device")
    L = kd.lib()
    cases = [dict(B=1, H=8, T=1152, seed=902, dtype="bf16"),            # 144 chunk-heads, tensor-core path
             dict(B=2, H=4, T=1000, seed=901, dtype="bf16"),            # 128 chunk-heads, ragged tail
             dict(B=2, H=3, T=300, dk=64, dv=64, seed=903, dtype="f32")]  # CUDA-core path, ragged tail
    for i, case in enumerate(cases):
        dt = case["dtype"]
        inp = kin.make_inputs(3, B=case["B"], H=case["H"], T=case["T"], dk=case.get("dk"), dv=case.get("dv"),
                              seed=case["seed"], with_dO=False)
        adt = torch.bfloat16 if dt == "bf16" else torch.float32
        d = {n: torch.from_numpy(inp[n]).to("cuda", adt if n in ("q", "k", "v") else torch.float32)
             for n in ("q", "k", "v", "beta", "c", "logf", "S0")}
        ref_out, ref_ST, _ = kd.fwd(d["q"], d["k"], d["v"], d["beta"], d["c"], d["logf"], d["S0"])
        code = kd.KD_BF16 if dt == "bf16" else kd.KD_F32
        for _ in range(2):  # two calls in a row on the shared array
            out, ST = _noalloc(L, d, code)
            assert torch.equal(out, ref_out) and torch.equal(ST, ref_ST), case
        if i == 1:
            O_or, ST_or = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["c"], inp["logf"], inp["S0"])
            for x, ref in ((out, O_or), (ST, ST_or)):
                x = x.double().cpu().numpy()
                assert np.isfinite(x).all()
                assert np.linalg.norm(x - ref) / np.linalg.norm(ref) <= TOL_BF16
