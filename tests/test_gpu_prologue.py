"""GPU parity of the input prologue (kron_delta_prologue_fwd / _bwd) against
the fp64 prologue oracle on identical seeded inputs, element by element.

Tolerances, from the arithmetic (fp32 inside the kernel, one rounding to the
storage dtype on the way out):
  * dtype outputs (q, k, v; dq~, dk~, dv~, df): the kernel rounds an fp32 value
    to the storage dtype once, so |x - ref| <= 2^-8 |ref| for bf16 (2^-23 for
    fp32) plus the fp32 error of the row arithmetic; that error is below
    1e-5 of the row's largest magnitude (a 128-term fp32 dot product, one
    rsqrt, a few products), which is the absolute slack allowed per row.
  * fp32 gates (beta, c, logf, dbeta~, dc~): a handful of correctly rounded or
    few-ulp operations: relative 1e-5, absolute 1e-7.
  * da_log: an fp32 sum of N*dk terms in a fixed tree; the rounding error is
    below 1e-5 of the sum of the terms' magnitudes.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import delta_rule_linear_kron_b200 as kd  # noqa: E402
from delta_rule_linear_kron_b200 import inputs as kin  # noqa: E402
from oracle import prologue as P  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    kd.lib()


RAW = ("q_raw", "k_raw", "v_raw", "f_pre")
F32 = ("beta_pre", "c_pre", "a_log", "dbeta", "dc", "dlogf")


def dev(inp, dtype):
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    return {n: torch.from_numpy(x).to("cuda", dtype=torch.float32 if n in F32 else tdt).contiguous()
            for n, x in inp.items()}


def host(t):
    return t.detach().double().cpu().numpy()


def close_rows(x, ref, dtype, name):
    """Elementwise: |x - ref| <= rel*|ref| + 1e-5 * max|ref| over the row (last axis)."""
    rel = 2.0 ** -8 if dtype == "bf16" else 2.0 ** -22
    slack = 1e-5 * np.max(np.abs(ref), axis=-1, keepdims=True) + 1e-30
    bad = np.abs(x - ref) > rel * np.abs(ref) + slack
    assert not bad.any(), f"{name}: {int(bad.sum())} elements off, worst at {np.argwhere(bad)[0]}"


def close_f32(x, ref, name, rel=1e-5, atol=1e-7):
    bad = np.abs(x - ref) > rel * np.abs(ref) + atol
    assert not bad.any(), f"{name}: {int(bad.sum())} elements off, worst at {np.argwhere(bad)[0]}"


def run(inp, dtype, beta_scale):
    d = dev(inp, dtype)
    o = kd.prologue_fwd(d["q_raw"], d["k_raw"], d["v_raw"], d["beta_pre"], d["c_pre"], d["f_pre"], d["a_log"],
                        beta_scale)
    g = kd.prologue_bwd(d["q_raw"], d["k_raw"], d["v_raw"], d["beta_pre"], d["c_pre"], d["f_pre"], d["a_log"],
                        d["dq"], d["dk"], d["dv"], d["dbeta"], d["dc"], d["dlogf"], beta_scale)
    torch.cuda.synchronize()
    return d, o, g


def check(inp, dtype, beta_scale):
    _, o, g = run(inp, dtype, beta_scale)
    raw = {n: inp[n] for n in ("q_raw", "k_raw", "v_raw", "beta_pre", "c_pre", "f_pre", "a_log")}
    ro = P.prologue_fwd(**raw, beta_scale=beta_scale)
    for n in ("q", "k", "v"):
        close_rows(host(o[n]), ro[n], dtype, n)
    for n in ("beta", "c", "logf"):
        close_f32(host(o[n]), ro[n], n)
    rg = P.prologue_bwd(**raw, dq=inp["dq"], dk=inp["dk"], dv=inp["dv"], dbeta=inp["dbeta"], dc=inp["dc"],
                        dlogf=inp["dlogf"], beta_scale=beta_scale)
    for n in ("dq_raw", "dk_raw", "dv_raw", "df_pre"):
        close_rows(host(g[n]), rg[n], dtype, n)
    for n in ("dbeta_pre", "dc_pre"):
        close_f32(host(g[n]), rg[n], n)
    a = np.exp(raw["a_log"])[None, None, :, None]
    mag = np.sum(np.abs(inp["dlogf"] * a * P.log_sigmoid(raw["f_pre"])), axis=(0, 1, 3))
    assert np.all(np.abs(host(g["da_log"]) - rg["da_log"]) <= 1e-5 * mag + 1e-7), (host(g["da_log"]), rg["da_log"])
    return o, g


@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_prologue_small(dk, dv, dtype):
    check(kin.make_prologue_inputs(2, 3, 77, dk, dv, dtype, seed=dk + dv), dtype, 1.0)


@pytest.mark.parametrize("T", [1, 63, 64, 65, 1000])
def test_prologue_ragged_lengths_state_tracking(T):
    """beta_scale = 2 (beta in (0,2)); token counts that leave partial blocks."""
    check(kin.make_prologue_inputs(1, 5, T, 128, 128, "bf16", seed=T), "bf16", 2.0)


def test_prologue_edge_values():
    """All-zero rows (normalised to zero, gradient r*g), saturated gates and
    forget pre-activations (log sigmoid at +-30), a_log = 0 and a large a_log."""
    inp = kin.make_prologue_inputs(1, 4, 130, 64, 64, "f32", seed=5)
    inp["q_raw"][0, 3, 1, :] = 0.0
    inp["v_raw"][0, 7, 2, :] = 0.0
    inp["f_pre"][0, :10, 0, :] = 30.0
    inp["f_pre"][0, 10:20, 0, :] = -30.0
    inp["beta_pre"][0, :5, :] = 40.0
    inp["c_pre"][0, :5, :] = -40.0
    inp["a_log"][:] = [0.0, 2.5, -3.0, 1.0]
    check(inp, "f32", 1.0)


def test_prologue_workload_B1_H16_T16384():
    """The full-size mixer workload (B=1, H=16, T=16384, d=128, bf16), every element."""
    check(kin.make_prologue_inputs(1, 16, 16384, 128, 128, "bf16", seed=2004), "bf16", 2.0)


def test_prologue_bwd_deterministic():
    inp = kin.make_prologue_inputs(2, 8, 3000, 128, 128, "bf16", seed=9)
    _, _, g1 = run(inp, "bf16", 1.0)
    _, _, g2 = run(inp, "bf16", 1.0)
    for n in g1:
        assert torch.equal(g1[n], g2[n]), n


def test_prologue_feeds_the_mixer(oracle):
    """Raw inputs -> prologue -> chunked forward, against the oracle's prologue
    followed by the oracle's recurrence on the same inputs (q, k, v rounded to
    bf16 in between, as the GPU stores them)."""
    inp = kin.make_prologue_inputs(1, 2, 200, 128, 128, "bf16", seed=12, with_grads=False)
    d = dev(inp, "bf16")
    o = kd.prologue_fwd(*(d[n] for n in ("q_raw", "k_raw", "v_raw", "beta_pre", "c_pre", "f_pre", "a_log")))
    out, ST, _ = kd.fwd(o["q"], o["k"], o["v"], o["beta"], o["c"], o["logf"])
    torch.cuda.synchronize()
    ro = P.prologue_fwd(**inp)
    q, k, v = (kin.round_to_dtype(ro[n], "bf16") for n in ("q", "k", "v"))
    O_ref, ST_ref = oracle.fwd(q, k, v, ro["beta"], ro["c"], ro["logf"])
    for x, ref in ((host(out), O_ref), (host(ST), ST_ref)):
        assert np.linalg.norm(x - ref) <= 5e-3 * np.linalg.norm(ref)


def test_prologue_and_epilogue_autograd_match_direct_calls():
    inp = kin.make_prologue_inputs(1, 3, 90, 64, 64, "f32", seed=21)
    d = dev(inp, "f32")
    names = ("q_raw", "k_raw", "v_raw", "beta_pre", "c_pre", "f_pre", "a_log")
    leaves = [d[n].clone().requires_grad_(True) for n in names]
    outs = kd.PrologueFunction.apply(*leaves, 2.0)
    ups = [d[n] for n in ("dq", "dk", "dv", "dbeta", "dc", "dlogf")]
    sum((o * u).sum() for o, u in zip(outs, ups)).backward()
    g = kd.prologue_bwd(*(d[n] for n in names), *ups, 2.0)
    for leaf, gn in zip(leaves, ("dq_raw", "dk_raw", "dv_raw", "dbeta_pre", "dc_pre", "df_pre", "da_log")):
        assert torch.equal(leaf.grad, g[gn]), gn
    e = kin.make_epilogue_inputs(1, 3, 90, 64, "f32", seed=22)
    et = {n: torch.from_numpy(x).float().cuda() for n, x in e.items()}
    el = [et[n].clone().requires_grad_(True) for n in ("o", "g", "w")]
    (kd.EpilogueFunction.apply(*el) * et["dy"]).sum().backward()
    r = kd.epilogue_bwd(et["o"], et["g"], et["w"], et["dy"])
    for leaf, gn in zip(el, ("dO", "dg", "dw")):
        assert torch.equal(leaf.grad, r[gn]), gn
