"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
identical seeded inputs.

Tolerances (relative L2 over each whole tensor, against the oracle):
  fp32 inputs: 1e-4 on O and S_T; bf16 inputs: 5e-3 on O and S_T;
  gradients: 1e-2 (bf16) and 1e-4 (fp32).
Full-size workloads run in the same launch configuration as bench.py.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import delta_rule_linear_kron_b200 as kd  # noqa: E402
from delta_rule_linear_kron_b200 import inputs as kin  # noqa: E402

TOL_F32, TOL_BF16, TOL_GRAD_BF16, TOL_GRAD_F32 = 1e-4, 5e-3, 1e-2, 1e-4


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    kd.lib()  # loud failure if the library is missing


def rel(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-300))


def rel_units(x, ref, axes):
    """Largest relative L2 error over the units left after reducing `axes`
    (for example one value per (b, h) of a [B, T, H, d] tensor)."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    num = np.sqrt(np.sum((x - ref) ** 2, axis=axes))
    den = np.maximum(np.sqrt(np.sum(ref ** 2, axis=axes)), 1e-300)
    return float(np.max(num / den))


# per-(b,h) reduction axes of each tensor: [B,T,H,d], [B,T,H] and [B,H,dv,dk]
UNIT_AXES = {"O": (1, 3), "ST": (2, 3), "dq": (1, 3), "dk": (1, 3), "dv": (1, 3), "dbeta": (1,), "dc": (1,),
             "dlogf": (1, 3), "dS0": (2, 3)}


def rel_chunks(x, ref, C=64):
    """Largest relative L2 error over (b, chunk, h) blocks of a [B, T, H, d]
    tensor whose T is a multiple of C."""
    B, T, H, d = np.shape(ref)
    sh = (B, T // C, C, H, d)
    return rel_units(np.reshape(x, sh), np.reshape(ref, sh), (2, 4))


def dev(inp, dtype):
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    out = {}
    for n in ("q", "k", "v", "dO"):
        if n in inp and inp[n] is not None:
            out[n] = torch.from_numpy(inp[n]).to("cuda", dtype=tdt).contiguous()
    for n in ("beta", "c", "logf", "S0"):
        out[n] = None if inp.get(n) is None else torch.from_numpy(inp[n]).to("cuda", dtype=torch.float32).contiguous()
    return out


def host(t):
    return t.detach().double().cpu().numpy()


def run_fwd(inp, dtype, save=False):
    d = dev(inp, dtype)
    out, ST, ws = kd.fwd(d["q"], d["k"], d["v"], d["beta"], d["c"], d["logf"], d["S0"], save=save)
    torch.cuda.synchronize()
    kd.device_status()
    return d, out, ST, ws


def check_fwd(inp, dtype, tol, oracle, per_unit=False):
    """Whole-tensor relative L2 errors of O and S_T; with per_unit, also the
    largest error over single (b, h) heads and over single 64-token chunks of O,
    at the same tolerance (so one wrong head or chunk cannot hide in the norm)."""
    d, out, ST, _ = run_fwd(inp, dtype)
    O_ref, ST_ref = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["c"], inp["logf"], inp["S0"])
    o, s = host(out), host(ST)
    eo, es = rel(o, O_ref), rel(s, ST_ref)
    assert eo <= tol and es <= tol, (eo, es)
    if per_unit:
        uo, us, co = rel_units(o, O_ref, UNIT_AXES["O"]), rel_units(s, ST_ref, UNIT_AXES["ST"]), rel_chunks(o, O_ref)
        assert uo <= tol and us <= tol and co <= tol, dict(O_head=uo, ST_head=us, O_chunk=co)
    return eo, es


# ----------------------------------------------------------------------------- decode
@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_small(oracle, dk, dv, dtype):
    d = kin.make_decode_inputs(3, B=3, H=2, dk=dk, dv=dv, dtype=dtype, seed=7)
    S = torch.from_numpy(d["S"]).float().cuda()
    Sref = d["S"]
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    for t in range(3):
        args = [torch.from_numpy(d[n][t]).cuda().to(tdt) for n in ("q", "k", "v")]
        args += [torch.from_numpy(d[n][t]).float().cuda() for n in ("beta", "c", "logf")]
        o = kd.decode(*args, S)
        Sref, oref = oracle.decode(d["q"][t], d["k"][t], d["v"][t], d["beta"][t], d["c"][t], d["logf"][t], Sref)
        assert rel(host(S), Sref) <= 1e-5
        assert rel(host(o), oref) <= (1e-5 if dtype == "f32" else TOL_BF16)


def test_decode_full_batch_first_steps(oracle):
    """Decode workload B=256, H=16, d=128: first 8 steps on every head."""
    steps = 8
    d = kin.make_decode_inputs(steps)
    S = torch.from_numpy(d["S"]).float().cuda()
    Sref = d["S"]
    for t in range(steps):
        args = [torch.from_numpy(d[n][t]).cuda().to(torch.bfloat16) for n in ("q", "k", "v")]
        args += [torch.from_numpy(d[n][t]).float().cuda() for n in ("beta", "c", "logf")]
        o = kd.decode(*args, S)
        Sref, oref = oracle.decode(d["q"][t], d["k"][t], d["v"][t], d["beta"][t], d["c"][t], d["logf"][t], Sref)
        oh, Sh = host(o), host(S)
        assert rel(oh, oref) <= TOL_BF16
        assert rel(Sh, Sref) <= TOL_BF16
        # every single head ([B, H, d] outputs, [B, H, dv, dk] states)
        assert rel_units(oh, oref, (2,)) <= TOL_BF16
        assert rel_units(Sh, Sref, (2, 3)) <= TOL_BF16


def test_decode_1000_steps_sampled_heads(oracle):
    """The benchmark's 1000 in-place steps (device-drawn inputs); the final
    state and last output are checked on 64 sampled heads."""
    steps = 1000
    d = kin.decode_token_inputs_torch(steps)
    S = d["S"].clone()
    S_init = host(d["S"])
    for t in range(steps):
        o = kd.decode(d["q"][t], d["k"][t], d["v"][t], d["beta"][t], d["c"][t], d["logf"][t], S)
    torch.cuda.synchronize()
    rng = np.random.default_rng(0)
    heads = rng.choice(256 * 16, size=64, replace=False)
    bi, hi = heads // 16, heads % 16
    sel = lambda x: host(x[:, bi, hi])  # noqa: E731
    q, k, v, beta, c, logf = (sel(d[n]) for n in ("q", "k", "v", "beta", "c", "logf"))
    Sref = S_init[bi, hi][None]
    for t in range(steps):
        Sref, oref = oracle.decode(q[t][None], k[t][None], v[t][None], beta[t][None], c[t][None], logf[t][None], Sref)
    assert rel(host(S)[bi, hi], Sref[0]) <= TOL_BF16
    assert rel(host(o)[bi, hi], oref[0]) <= TOL_BF16
    assert rel_units(host(S)[bi, hi], Sref[0], (1, 2)) <= TOL_BF16
    assert rel_units(host(o)[bi, hi], oref[0], (1,)) <= TOL_BF16


# ----------------------------------------------------------------------------- forward
def test_fwd_tiny_fp32_workload(oracle):
    check_fwd(kin.make_inputs(1), "f32", TOL_F32, oracle)


@pytest.mark.parametrize("T", [1, 63, 64, 65, 200])
@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64), ("bf16", 32)])
def test_fwd_small_ragged(oracle, T, dtype, d):
    inp = kin.make_inputs(3, B=2, H=3, T=T, dk=d, dv=d, seed=100 + T)
    inp["wl"] = None
    check_fwd(inp, dtype, TOL_F32 if dtype == "f32" else TOL_BF16, oracle)


def test_fwd_rectangular_state(oracle):
    inp = kin.make_inputs(3, B=1, H=2, T=150, dk=128, dv=64, seed=5)
    check_fwd(inp, "bf16", TOL_BF16, oracle)
    inp = kin.make_inputs(3, B=1, H=2, T=150, dk=32, dv=128, seed=6)
    check_fwd(inp, "f32", TOL_F32, oracle)


def test_fwd_workload_B4_T2048(oracle):
    check_fwd(kin.make_inputs(2, with_dO=False), "bf16", TOL_BF16, oracle, per_unit=True)


def test_fwd_workload_T16384_nonzero_state(oracle):
    check_fwd(kin.make_inputs(3, with_dO=False), "bf16", TOL_BF16, oracle, per_unit=True)


@pytest.mark.parametrize("beta_val", [0.0, 1.0])
def test_fwd_beta_edges(oracle, beta_val):
    inp = kin.make_inputs(1, T=150, seed=9)
    inp["beta"] = np.full_like(inp["beta"], beta_val)
    check_fwd(inp, "f32", TOL_F32, oracle)


def _extreme(inp, seed):
    rng = np.random.default_rng(seed)
    lf = inp["logf"].copy()
    B, T, H, dk = lf.shape
    for _ in range(6):  # bursts of strong decay in random channels
        t0 = rng.integers(0, max(1, T - 8))
        ch = rng.choice(dk, size=dk // 4, replace=False)
        lf[:, t0:t0 + 8, :, :][..., ch] = -30.0 - 10.0 * rng.random()
    inp["logf"] = kin.round_to_dtype(lf, "f32")
    return inp


@pytest.mark.parametrize("dtype,d", [("f32", 32), ("bf16", 128)])
def test_fwd_extreme_decay(oracle, dtype, d):
    inp = _extreme(kin.make_inputs(3, B=1, H=2, T=200, dk=d, dv=d, seed=11), 3)
    check_fwd(inp, dtype, TOL_F32 if dtype == "f32" else TOL_BF16, oracle)


def test_decode_steps_match_chunked_fwd():
    inp = kin.make_inputs(3, B=2, H=2, T=100, dk=64, dv=64, seed=21)
    d, out, ST, _ = run_fwd(inp, "f32")
    S = d["S0"].clone()
    outs = []
    for t in range(100):
        outs.append(kd.decode(d["q"][:, t].contiguous(), d["k"][:, t].contiguous(), d["v"][:, t].contiguous(),
                              d["beta"][:, t].contiguous(), d["c"][:, t].contiguous(),
                              d["logf"][:, t].contiguous(), S))
    torch.cuda.synchronize()
    assert rel(host(torch.stack(outs, 1)), host(out)) <= 1e-5
    assert rel(host(S), host(ST)) <= 1e-5


def test_fwd_deterministic():
    inp = kin.make_inputs(3, B=1, H=4, T=300, seed=31)
    _, o1, s1, _ = run_fwd(inp, "bf16")
    _, o2, s2, _ = run_fwd(inp, "bf16")
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


# ----------------------------------------------------------------------------- backward
GRADS = ("dq", "dk", "dv", "dbeta", "dc", "dlogf", "dS0")


def check_bwd(inp, dtype, tol_fwd, tol_grad, oracle, dST=None, per_unit=False):
    """Forward and every gradient against the oracle (whole-tensor relative L2);
    with per_unit, also per (b, h) head for every tensor and per 64-token chunk
    for O, dq, dk and dv, at the same tolerances."""
    d, out, ST, ws = run_fwd(inp, dtype, save=True)
    dSTd = None if dST is None else torch.from_numpy(dST).float().cuda()
    g = kd.bwd(d["q"], d["k"], d["v"], d["beta"], d["c"], d["logf"], d["S0"], d["dO"], dSTd, fwd_workspace=ws)
    torch.cuda.synchronize()
    kd.device_status()
    O_ref, ST_ref = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["c"], inp["logf"], inp["S0"])
    assert rel(host(out), O_ref) <= tol_fwd and rel(host(ST), ST_ref) <= tol_fwd
    gr = oracle.bwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["c"], inp["logf"], inp["S0"], inp["dO"], dST)
    gh = {n: host(g[n]) for n in GRADS}
    errs = {n: rel(gh[n], gr[n]) for n in GRADS}
    assert all(e <= tol_grad for e in errs.values()), errs
    if per_unit:
        o = host(out)
        fw = dict(O_head=rel_units(o, O_ref, UNIT_AXES["O"]), ST_head=rel_units(host(ST), ST_ref, UNIT_AXES["ST"]),
                  O_chunk=rel_chunks(o, O_ref))
        assert all(e <= tol_fwd for e in fw.values()), fw
        heads = {n: rel_units(gh[n], gr[n], UNIT_AXES[n]) for n in GRADS}
        assert all(e <= tol_grad for e in heads.values()), heads
        chunks = {n: rel_chunks(gh[n], gr[n]) for n in ("dq", "dk", "dv")}
        assert all(e <= tol_grad for e in chunks.values()), chunks
    return errs


@pytest.mark.parametrize("T", [64, 150])
def test_bwd_small_fp32(oracle, T):
    inp = kin.make_inputs(4, B=1, H=2, T=T, dk=32, dv=32, seed=40 + T)
    dST = np.random.default_rng(T).standard_normal((1, 2, 32, 32))
    check_bwd(inp, "f32", TOL_F32, TOL_GRAD_F32, oracle, dST)


@pytest.mark.parametrize("T", [1, 100, 256])
def test_bwd_small_bf16(oracle, T):
    inp = kin.make_inputs(4, B=2, H=2, T=T, seed=50 + T)
    check_bwd(inp, "bf16", TOL_BF16, TOL_GRAD_BF16, oracle)


def test_bwd_zero_initial_state_and_dST(oracle):
    inp = kin.make_inputs(4, B=1, H=2, T=130, dk=64, dv=64, seed=61, s0="zero")
    dST = np.random.default_rng(1).standard_normal((1, 2, 64, 64))
    check_bwd(inp, "f32", TOL_F32, TOL_GRAD_F32, oracle, dST)


@pytest.mark.parametrize("dtype,d", [("f32", 32), ("bf16", 128)])
def test_bwd_extreme_decay(oracle, dtype, d):
    inp = _extreme(kin.make_inputs(4, B=1, H=2, T=200, dk=d, dv=d, seed=71), 4)
    check_bwd(inp, dtype, TOL_F32 if dtype == "f32" else TOL_BF16,
              TOL_GRAD_F32 if dtype == "f32" else TOL_GRAD_BF16, oracle)


def test_bwd_bf16_ragged_with_dST(oracle):
    """Tensor-core backward with a nonzero final-state gradient and a ragged tail."""
    inp = kin.make_inputs(4, B=1, H=3, T=130, seed=91)
    dST = np.random.default_rng(5).standard_normal((1, 3, 128, 128)) / 128.0
    check_bwd(inp, "bf16", TOL_BF16, TOL_GRAD_BF16, oracle, dST)


def test_bwd_bf16_decay_bands(oracle):
    """Heads whose in-chunk cumulative decay stays mild, reaches the 40..80
    band (tensor-core pre-chain products, exact post-chain path) and goes
    beyond it (exact path throughout)."""
    inp = kin.make_inputs(4, B=1, H=3, T=200, seed=92)
    lf = inp["logf"].copy()
    lf[:, :, 1, :] = -0.9                     # |L| up to ~57 inside a chunk
    lf[:, :, 2, :] = np.minimum(lf[:, :, 2, :] * 30.0, -1.5)  # |L| far beyond 80
    inp["logf"] = kin.round_to_dtype(lf, "f32")
    check_bwd(inp, "bf16", TOL_BF16, TOL_GRAD_BF16, oracle)


def test_fwdbwd_workload_T16384_state_tracking(oracle):
    """Forward+backward workload: B=1, H=16, T=16384, d=128, beta in (0,2)."""
    check_bwd(kin.make_inputs(4), "bf16", TOL_BF16, TOL_GRAD_BF16, oracle, per_unit=True)


def test_autograd_function_matches_bwd():
    inp = kin.make_inputs(4, B=1, H=2, T=70, dk=32, dv=32, seed=81)
    d = dev(inp, "f32")
    leaves = {n: d[n].clone().requires_grad_(True) for n in ("q", "k", "v", "beta", "c", "logf", "S0")}
    out, ST = kd.KronDeltaFunction.apply(*(leaves[n] for n in ("q", "k", "v", "beta", "c", "logf", "S0")))
    (out * d["dO"]).sum().backward()
    _, _, _, ws = run_fwd(inp, "f32", save=True)
    g = kd.bwd(d["q"], d["k"], d["v"], d["beta"], d["c"], d["logf"], d["S0"], d["dO"], fwd_workspace=ws)
    for n, gn in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("beta", "dbeta"), ("c", "dc"), ("logf", "dlogf"),
                  ("S0", "dS0")):
        assert torch.allclose(leaves[n].grad, g[gn], rtol=1e-6, atol=1e-7), n
