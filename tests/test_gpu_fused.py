"""GPU parity of the fused entry points (kron_delta_fwd_fused / _bwd_fused:
raw q, k, v projections and gate pre-activations, the input prologue inside
the chunk kernels) against the fp64 oracles composed: oracle/prologue.py
forms q, k, v, beta, c, logf from the raw inputs (q, k, v then stored in the
activation dtype, as the library's prologue stores them and as the fused
kernels hold them), oracle/kd_oracle.c runs the recurrence and its
reverse-mode, and oracle/prologue.py's backward carries the gradients back to
the raw inputs.

Tolerances as for the plain path (relative L2 against the oracle): bf16 5e-3
on O and S_T and 1e-2 on every gradient; fp32 1e-4 throughout.  da_log, a
sum over tokens and channels whose terms cancel, is held to the same numbers
relative to the sum of its terms' magnitudes.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import delta_rule_linear_kron_b200 as kd  # noqa: E402
from delta_rule_linear_kron_b200 import inputs as kin  # noqa: E402
from oracle import prologue as P  # noqa: E402

TOL = {"f32": (1e-4, 1e-4), "bf16": (5e-3, 1e-2)}
RAW = ("q_raw", "k_raw", "v_raw", "beta_pre", "c_pre", "f_pre", "a_log")


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


def make(B, H, T, d, dtype, seed, s0=True, with_dST=False):
    inp = kin.make_prologue_inputs(B, H, T, d, d, dtype, seed=seed, with_grads=False)
    rng = np.random.default_rng(seed + 1)
    inp["dO"] = kin.round_to_dtype(rng.standard_normal((B, T, H, d)), dtype)
    inp["S0"] = rng.standard_normal((B, H, d, d)) / d if s0 else None
    inp["dST"] = rng.standard_normal((B, H, d, d)) / d if with_dST else None
    return inp


def check(inp, dtype, oracle, beta_scale, per_head=False):
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    d = {n: torch.from_numpy(inp[n]).to("cuda", tdt) for n in ("q_raw", "k_raw", "v_raw", "f_pre", "dO")}
    for n in ("beta_pre", "c_pre", "a_log"):
        d[n] = torch.from_numpy(inp[n]).to("cuda", torch.float32)
    d["S0"] = None if inp["S0"] is None else torch.from_numpy(inp["S0"]).to("cuda", torch.float32)
    dST = None if inp["dST"] is None else torch.from_numpy(inp["dST"]).to("cuda", torch.float32)
    raw = [d[n] for n in RAW]
    out, ST, ws = kd.fwd_fused(*raw, beta_scale, d["S0"], save=True)
    g = kd.bwd_fused(*raw, beta_scale, d["S0"], d["dO"], dST, fwd_workspace=ws)
    torch.cuda.synchronize()
    kd.device_status()

    # the composition the fused path stands for: the prologue, whose q, k, v
    # outputs are stored in the activation dtype, then the recurrence
    pro = P.prologue_fwd(*(inp[n] for n in RAW), beta_scale=beta_scale)
    for n in ("q", "k", "v"):
        pro[n] = kin.round_to_dtype(pro[n], dtype)
    args = [pro[n] for n in ("q", "k", "v", "beta", "c", "logf")]
    O_ref, ST_ref = oracle.fwd(*args, inp["S0"])
    gr = oracle.bwd(*args, inp["S0"], inp["dO"], inp["dST"])
    pb = P.prologue_bwd(*(inp[n] for n in RAW), gr["dq"], gr["dk"], gr["dv"], gr["dbeta"], gr["dc"], gr["dlogf"],
                        beta_scale=beta_scale)
    tf, tg = TOL[dtype]
    errs = {"O": rel(host(out), O_ref), "ST": rel(host(ST), ST_ref), "dS0": rel(host(g["dS0"]), gr["dS0"])}
    for n in ("dq_raw", "dk_raw", "dv_raw", "dbeta_pre", "dc_pre", "df_pre"):
        errs[n] = rel(host(g[n]), pb[n])
    # da_log[h] = sum over tokens and key channels of dlogf logf: a sum whose
    # terms cancel, so its error is held against the sum of the terms' sizes
    scale = np.sum(np.abs(gr["dlogf"] * pro["logf"]), axis=(0, 1, 3))
    errs["da_log"] = float(np.max(np.abs(host(g["da_log"]) - pb["da_log"]) / scale))
    bad = {n: e for n, e in errs.items() if e > (tf if n in ("O", "ST") else tg)}
    assert not bad, errs
    if per_head:
        H = inp["q_raw"].shape[2]
        for h in range(H):
            one = {"O": rel(host(out)[:, :, h], O_ref[:, :, h])}
            for n in ("dq_raw", "dk_raw", "dv_raw", "df_pre"):
                one[n] = rel(host(g[n])[:, :, h], pb[n][:, :, h])
            # per head, df_pre gets twice the gradient tolerance: it weights
            # dlogf by a sigma(-f_pre), largest where the decay is strongest,
            # which is where dlogf's decay-weighted reverse sums carry their
            # largest errors (the unfused prologue + recurrence path measures
            # the same per-head figure); a wrong head is still off by O(1)
            bad = {n: e for n, e in one.items() if e > (tf if n == "O" else 2 * tg if n == "df_pre" else tg)}
            assert not bad, (h, one)
    return errs


def test_fused_tensor_core_ragged(oracle):
    check(make(1, 3, 150, 128, "bf16", 501, with_dST=True), "bf16", oracle, 2.0)


def test_fused_tensor_core_zero_state(oracle):
    check(make(2, 2, 64, 128, "bf16", 503, s0=False), "bf16", oracle, 1.0)


def test_fused_cuda_core_fp32(oracle):
    check(make(2, 2, 100, 32, "f32", 505), "f32", oracle, 1.0)


def test_fused_cuda_core_bf16_d64(oracle):
    check(make(1, 2, 130, 64, "bf16", 507, with_dST=True), "bf16", oracle, 2.0)


def test_fused_extreme_decay_exact_paths(oracle):
    """Bursts of saturated forget pre-activations: chunks beyond the factorised
    range take the exact paths, which read the normalised rows the preparation
    kernel kept for them."""
    inp = make(1, 2, 200, 128, "bf16", 509)
    rng = np.random.default_rng(9)
    fp = inp["f_pre"].copy()
    for _ in range(6):
        t0 = rng.integers(0, 192)
        ch = rng.choice(128, size=32, replace=False)
        fp[:, t0:t0 + 8, :, :][..., ch] = -30.0 - 10.0 * rng.random()
    inp["f_pre"] = kin.round_to_dtype(fp, "bf16")
    check(inp, "bf16", oracle, 2.0)


def test_fused_workload_T16384(oracle):
    """The forward+backward workload's shape (B=1, H=16, T=16384, d=128, bf16,
    beta in (0,2)) from raw inputs: every head checked."""
    check(make(1, 16, 16384, 128, "bf16", 511), "bf16", oracle, 2.0, per_head=True)
