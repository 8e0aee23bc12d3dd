"""GPU parity of the Gated DeltaNet-2 kernels (kron_delta_gdn2_fwd / _bwd)
against the fp64 token oracle (oracle/gdn2.py) on identical seeded inputs.

Tolerances (relative L2 over each tensor, as for the Kronecker rule): fp32
inputs 1e-4 on outputs, states and gradients; bf16 inputs 5e-3 on O and S_T
and 1e-2 on gradients (the kernels compute in fp32; the error is the bf16
rounding of O and of the stored gradients).  The full-size case checks
sampled heads: every head is independent, so the oracle runs on those heads'
slices alone.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import delta_rule_linear_kron_b200 as kd  # noqa: E402
from delta_rule_linear_kron_b200 import inputs as kin  # noqa: E402
from oracle import gdn2 as G  # noqa: E402

TOL = {"f32": (1e-4, 1e-4), "bf16": (5e-3, 1e-2)}
NAMES = ("q", "k", "v", "b", "w", "loga")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    kd.lib()


def rel(x, ref):
    return float(np.linalg.norm(np.asarray(x, dtype=np.float64) - ref) / max(np.linalg.norm(ref), 1e-300))


def dev(inp, dtype):
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    d = {}
    for n in ("q", "k", "v", "dO"):
        d[n] = torch.from_numpy(inp[n]).to("cuda", dtype=tdt).contiguous()
    for n in ("b", "w", "loga"):
        d[n] = torch.from_numpy(inp[n]).to("cuda", dtype=torch.float32).contiguous()
    d["S0"] = None if inp["S0"] is None else torch.from_numpy(inp["S0"]).float().cuda()
    return d


def host(t):
    return t.detach().double().cpu().numpy()


def run(inp, dtype, dST=None):
    d = dev(inp, dtype)
    out, ST, ws = kd.gdn2_fwd(*(d[n] for n in NAMES), d["S0"])
    dSTd = None if dST is None else torch.from_numpy(dST).float().cuda()
    g = kd.gdn2_bwd(*(d[n] for n in NAMES), d["S0"], d["dO"], dSTd, fwd_workspace=ws)
    torch.cuda.synchronize()
    kd.device_status()
    return out, ST, g


def check(inp, dtype, dST=None, heads=None):
    out, ST, g = run(inp, dtype, dST)
    sl = slice(None) if heads is None else heads
    ref_in = {n: inp[n][:, :, sl] for n in NAMES}
    S0 = None if inp["S0"] is None else inp["S0"][:, sl]
    dSTs = None if dST is None else dST[:, sl]
    O_ref, ST_ref = G.fwd(**ref_in, S0=S0)
    gr = G.bwd(**ref_in, S0=S0, dO=inp["dO"][:, :, sl], dST=dSTs)
    tf, tg = TOL[dtype]
    errs = {"O": rel(host(out)[:, :, sl], O_ref), "ST": rel(host(ST)[:, sl], ST_ref)}
    for n in ("dq", "dk", "dv", "db", "dw", "dloga"):
        errs[n] = rel(host(g[n])[:, :, sl], gr[n])
    errs["dS0"] = rel(host(g["dS0"])[:, sl], gr["dS0"])
    bad = {n: e for n, e in errs.items() if e > (tf if n in ("O", "ST") else tg)}
    assert not bad, errs
    if heads is not None:
        # each checked head on its own, at the same tolerances
        for j, hh in enumerate(heads):
            one = {"O": rel(host(out)[:, :, hh], O_ref[:, :, j]), "ST": rel(host(ST)[:, hh], ST_ref[:, j]),
                   "dS0": rel(host(g["dS0"])[:, hh], gr["dS0"][:, j])}
            for n in ("dq", "dk", "dv", "db", "dw", "dloga"):
                one[n] = rel(host(g[n])[:, :, hh], gr[n][:, :, j])
            bad = {n: e for n, e in one.items() if e > (tf if n in ("O", "ST") else tg)}
            assert not bad, (hh, one)
    return errs


@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_gdn2_small(dk, dv, dtype):
    check(kin.make_gdn2_inputs(1, 2, 150, dk, dv, dtype, seed=dk * 3 + dv), dtype)


@pytest.mark.parametrize("T", [1, 63, 64, 65, 200])
def test_gdn2_ragged_with_final_state_gradient(T):
    inp = kin.make_gdn2_inputs(2, 2, T, 64, 64, "f32", seed=T)
    dST = np.random.default_rng(T).standard_normal((2, 2, 64, 64)) / 64
    check(inp, "f32", dST)


def test_gdn2_zero_state_and_gated_delta_special_case():
    """S0 = 0 and b = w = beta (the gated delta rule the article recovers)."""
    inp = kin.make_gdn2_inputs(1, 2, 130, 32, 32, "f32", seed=7, s0="zero")
    beta = inp["b"][..., :1]
    inp["b"] = np.repeat(beta, 32, axis=-1)
    inp["w"] = np.repeat(beta, 32, axis=-1)
    check(inp, "f32")


def test_gdn2_extreme_decay():
    """Channels whose decay empties the state within a few tokens (|L| far
    beyond fp32's exponent range inside a chunk): the per-element weights keep
    every factor <= 1."""
    inp = kin.make_gdn2_inputs(1, 2, 200, 64, 64, "f32", seed=8)
    inp["loga"][:, :, 0, :8] = -30.0
    inp["loga"][:, :, 1, :] *= 40.0
    inp["loga"] = kin.round_to_dtype(inp["loga"], "f32")
    check(inp, "f32")


def test_gdn2_extreme_decay_tensor_cores():
    """The same extreme decays on the tensor-core preparation (bf16, d = 128):
    chunks whose in-chunk |L| reaches its factorised range take per-element
    weights, the others the tf32 products; both in one problem."""
    inp = kin.make_gdn2_inputs(1, 2, 260, 128, 128, "bf16", seed=18)
    inp["loga"][:, 70:78, 0, :8] = -30.0
    inp["loga"][:, :, 1, :] *= 40.0
    inp["loga"] = kin.round_to_dtype(inp["loga"], "f32")
    check(inp, "bf16")


def test_gdn2_tensor_cores_batched_ragged_with_final_state_gradient():
    """The tensor-core path (bf16, d = 128) with two batch entries, a ragged last
    chunk and a final-state gradient: every (b, h) checked on its own."""
    inp = kin.make_gdn2_inputs(2, 3, 200, 128, 128, "bf16", seed=71)
    dST = np.random.default_rng(72).standard_normal((2, 3, 128, 128)) / 128
    out, ST, g = run(inp, "bf16", dST)
    O_ref, ST_ref = G.fwd(**{n: inp[n] for n in NAMES}, S0=inp["S0"])
    gr = G.bwd(**{n: inp[n] for n in NAMES}, S0=inp["S0"], dO=inp["dO"], dST=dST)
    tf, tg = TOL["bf16"]
    for bb in range(2):
        for hh in range(3):
            one = {"O": rel(host(out)[bb, :, hh], O_ref[bb, :, hh]), "ST": rel(host(ST)[bb, hh], ST_ref[bb, hh]),
                   "dS0": rel(host(g["dS0"])[bb, hh], gr["dS0"][bb, hh])}
            for n in ("dq", "dk", "dv", "db", "dw", "dloga"):
                one[n] = rel(host(g[n])[bb, :, hh], gr[n][bb, :, hh])
            bad = {n: e for n, e in one.items() if e > (tf if n in ("O", "ST") else tg)}
            assert not bad, (bb, hh, one)


def test_gdn2_workload_B1_H16_T16384_sampled_heads():
    """The mixer's full-size shape (B=1, H=16, T=16384, d=128, bf16), run whole
    on the GPU; heads 0 and 11 checked against the oracle."""
    inp = kin.make_gdn2_inputs(1, 16, 16384, 128, 128, "bf16", seed=4004)
    check(inp, "bf16", heads=[0, 11])


def test_gdn2_deterministic():
    inp = kin.make_gdn2_inputs(1, 4, 300, 128, 128, "bf16", seed=9)
    o1, s1, g1 = run(inp, "bf16")
    o2, s2, g2 = run(inp, "bf16")
    assert torch.equal(o1, o2) and torch.equal(s1, s2)
    for n in g1:
        assert torch.equal(g1[n], g2[n]), n


@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_gdn2_decode_step(dk, dv, dtype):
    """One decode step against the oracle's one-token forward from the same state."""
    inp = kin.make_gdn2_inputs(4, 3, 1, dk, dv, dtype, seed=dk + 2 * dv)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    q, k, v = (torch.from_numpy(inp[n][:, 0]).to("cuda", dtype=tdt) for n in ("q", "k", "v"))
    b, w, loga = (torch.from_numpy(inp[n][:, 0]).float().cuda() for n in ("b", "w", "loga"))
    S = torch.from_numpy(inp["S0"]).float().cuda()
    o = kd.gdn2_decode(q, k, v, b, w, loga, S)
    torch.cuda.synchronize()
    O_ref, S_ref = G.fwd(**{n: inp[n] for n in NAMES}, S0=inp["S0"])
    tf = TOL[dtype][0]
    assert rel(host(o), O_ref[:, 0]) <= tf
    assert rel(host(S), S_ref) <= 1e-6


def test_gdn2_decode_steps_match_chunked_forward():
    """100 consecutive decode steps equal the chunked forward over the same 100 tokens."""
    inp = kin.make_gdn2_inputs(2, 4, 100, 128, 128, "bf16", seed=33)
    d = dev(inp, "bf16")
    out, ST, _ = kd.gdn2_fwd(*(d[n] for n in NAMES), d["S0"])
    S = d["S0"].clone()
    outs = []
    for t in range(100):
        outs.append(kd.gdn2_decode(*(d[n][:, t].contiguous() for n in NAMES), S))
    torch.cuda.synchronize()
    dec = torch.stack(outs, dim=1)
    assert rel(host(dec), host(out)) <= 5e-3
    assert rel(host(S), host(ST)) <= 1e-4


def test_gdn2_autograd_matches_direct_calls():
    inp = kin.make_gdn2_inputs(1, 2, 130, 64, 64, "f32", seed=44)
    d = dev(inp, "f32")
    leaves = [d[n].clone().requires_grad_(True) for n in (*NAMES, "S0")]
    out, ST = kd.Gdn2Function.apply(*leaves)
    (out * d["dO"]).sum().backward()
    _, _, ws = kd.gdn2_fwd(*(d[n] for n in NAMES), d["S0"])
    g = kd.gdn2_bwd(*(d[n] for n in NAMES), d["S0"], d["dO"], fwd_workspace=ws)
    for leaf, gn in zip(leaves, ("dq", "dk", "dv", "db", "dw", "dloga", "dS0")):
        assert torch.equal(leaf.grad, g[gn]), gn
