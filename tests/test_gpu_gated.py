"""GPU parity of the gated entry points (kron_delta_fwd_gated / _bwd_gated:
the forget gate given as its pre-activation f~ and the per-head exponent
a_log) against the fp64 oracles composed: oracle/prologue.py forms
logf = e^{a_log} log sigma(f~) and, in the backward, df~ and da_log from
dlogf; oracle/kd_oracle.c runs the recurrence and its reverse-mode.

Tolerances as for the plain path (relative L2 against the oracle): bf16
inputs 5e-3 on O and S_T and 1e-2 on every gradient (df~ and da_log
included); fp32 inputs 1e-4 throughout.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import delta_rule_linear_kron_b200 as kd  # noqa: E402
from delta_rule_linear_kron_b200 import inputs as kin  # noqa: E402
from oracle import prologue as P  # noqa: E402

TOL = {"f32": (1e-4, 1e-4), "bf16": (5e-3, 1e-2)}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    kd.lib()


def rel(x, ref):
    x = np.asarray(x, dtype=np.float64)
    return float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-300))


def host(t):
    return t.detach().double().cpu().numpy()


def oracle_gate(inp):
    """logf from the prologue oracle (its other outputs unused here)."""
    B, T, H, _ = inp["q"].shape
    z = np.zeros((B, T, H))
    return P.prologue_fwd(inp["q"], inp["k"], inp["v"], z, z, inp["f_pre"], inp["a_log"])["logf"]


def oracle_gate_bwd(inp, dlogf):
    """df~ and da_log from dlogf through the prologue oracle's backward."""
    B, T, H, dk = inp["q"].shape
    dv = inp["v"].shape[-1]
    z3, zk, zv = np.zeros((B, T, H)), np.zeros((B, T, H, dk)), np.zeros((B, T, H, dv))
    out = P.prologue_bwd(inp["q"], inp["k"], inp["v"], z3, z3, inp["f_pre"], inp["a_log"], zk, zk, zv, z3, z3,
                         dlogf)
    return out["df_pre"], out["da_log"]


def check(inp, dtype, oracle, dST=None, per_head=False):
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    d = {n: torch.from_numpy(inp[n]).to("cuda", tdt) for n in ("q", "k", "v", "dO", "f_pre")}
    for n in ("beta", "c", "a_log"):
        d[n] = torch.from_numpy(inp[n]).to("cuda", torch.float32)
    d["S0"] = None if inp["S0"] is None else torch.from_numpy(inp["S0"]).to("cuda", torch.float32)
    out, ST, ws = kd.fwd_gated(d["q"], d["k"], d["v"], d["beta"], d["c"], d["f_pre"], d["a_log"], d["S0"], save=True)
    dSTd = None if dST is None else torch.from_numpy(dST).to("cuda", torch.float32)
    g = kd.bwd_gated(d["q"], d["k"], d["v"], d["beta"], d["c"], d["f_pre"], d["a_log"], d["S0"], d["dO"], dSTd,
                     fwd_workspace=ws)
    torch.cuda.synchronize()
    kd.device_status()
    logf = oracle_gate(inp)
    O_ref, ST_ref = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["c"], logf, inp["S0"])
    gr = oracle.bwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["c"], logf, inp["S0"], inp["dO"], dST)
    df_ref, da_ref = oracle_gate_bwd(inp, gr["dlogf"])
    tf, tg = TOL[dtype]
    errs = {"O": rel(host(out), O_ref), "ST": rel(host(ST), ST_ref), "df_pre": rel(host(g["df_pre"]), df_ref),
            "da_log": rel(host(g["da_log"]), da_ref)}
    for n in ("dq", "dk", "dv", "dbeta", "dc", "dS0"):
        errs[n] = rel(host(g[n]), gr[n])
    bad = {n: e for n, e in errs.items() if e > (tf if n in ("O", "ST") else tg)}
    assert not bad, errs
    if per_head:
        H = inp["q"].shape[2]
        for h in range(H):
            one = {"O": rel(host(out)[:, :, h], O_ref[:, :, h]), "df_pre": rel(host(g["df_pre"])[:, :, h],
                                                                               df_ref[:, :, h])}
            for n in ("dq", "dk", "dv"):
                one[n] = rel(host(g[n])[:, :, h], gr[n][:, :, h])
            bad = {n: e for n, e in one.items() if e > (tf if n == "O" else tg)}
            assert not bad, (h, one)
    return errs


def test_gated_tensor_core_ragged(oracle):
    inp = kin.make_gated_inputs(4, B=1, H=3, T=150, seed=301, seed_gate=302)
    dST = np.random.default_rng(3).standard_normal((1, 3, 128, 128)) / 128.0
    check(inp, "bf16", oracle, dST)


def test_gated_cuda_core_fp32(oracle):
    inp = kin.make_gated_inputs(1, B=2, H=2, T=100, seed=303, seed_gate=304)
    inp["dO"] = np.random.default_rng(5).standard_normal(inp["q"].shape[:3] + (32,))
    check(inp, "f32", oracle)


def test_gated_extreme_decay_exact_paths(oracle):
    """Bursts of saturated forget pre-activations (log-decays near -30 a per
    token): chunks beyond the factorised range take the exact paths, which
    form the gate from its pre-activation too."""
    inp = kin.make_gated_inputs(4, B=1, H=2, T=200, seed=305, seed_gate=306)
    rng = np.random.default_rng(7)
    fp = inp["f_pre"].copy()
    for _ in range(6):
        t0 = rng.integers(0, 192)
        ch = rng.choice(128, size=32, replace=False)
        fp[:, t0:t0 + 8, :, :][..., ch] = -30.0 - 10.0 * rng.random()
    inp["f_pre"] = kin.round_to_dtype(fp, "bf16")
    check(inp, "bf16", oracle)


def test_gated_workload_T16384(oracle):
    """The forward+backward workload's shape (B=1, H=16, T=16384, d=128, bf16,
    beta in (0,2)) with the gate's pre-activations: every head checked."""
    check(kin.make_gated_inputs(4, seed_gate=3004), "bf16", oracle, per_head=True)
