"""GPU checks of the forward/backward phase split (kron_delta_fwd_phase /
kron_delta_bwd_phase) and of the context-parallel relay built on it.

* LOCAL then CARRY gives bitwise the result of one ALL call (same kernels, same
  order), on the tensor-core path and the general path.
* Time segments on one GPU, with every segment's LOCAL phase enqueued before
  any CARRY phase (the order a relay produces), and the state handed from one
  segment to the next by a device copy, equal the oracle on the whole sequence.
* relay_fwd / relay_bwd with the CUDA segment operations, as two processes over
  gloo sharing this GPU (the state crosses through host memory; the kernels of
  the two processes never wait on one another), equal the oracle too.
"""
import json
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import delta_rule_linear_kron_b200 as kd  # noqa: E402
from delta_rule_linear_kron_b200 import inputs as kin  # noqa: E402

TOL = {"bf16": (5e-3, 1e-2), "f32": (1e-4, 1e-4)}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    kd.lib()


def dev(inp, dtype, lo=0, hi=None):
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    out = {}
    for n in ("q", "k", "v", "dO", "beta", "c", "logf"):
        x = np.ascontiguousarray(inp[n][:, lo:hi])
        out[n] = torch.from_numpy(x).to("cuda", dtype=tdt if n in ("q", "k", "v", "dO") else torch.float32)
    out["S0"] = None if inp["S0"] is None else torch.from_numpy(inp["S0"]).float().cuda()
    return out


def host(t):
    return t.detach().double().cpu().numpy()


def rel(x, ref):
    return float(np.linalg.norm(np.asarray(x) - ref) / max(np.linalg.norm(ref), 1e-300))


ARGS = ("q", "k", "v", "beta", "c", "logf")


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 32)])
def test_phase_split_is_bitwise_the_whole_call(dtype, d):
    inp = kin.make_inputs(4, B=1, H=3, T=200, dk=d, dv=d, seed=5)
    x = dev(inp, dtype)
    a = [x[n] for n in ARGS]
    out1, ST1, ws1 = kd.fwd(*a, x["S0"], save=True)
    g1 = kd.bwd(*a, x["S0"], x["dO"], fwd_workspace=ws1)
    out2, ST2, ws2 = kd.fwd(*a, None, save=True, phase=kd.KD_PHASE_LOCAL)
    out2, ST2, _ = kd.fwd(*a, x["S0"], out=out2, state_out=ST2, save=True, workspace=ws2, phase=kd.KD_PHASE_CARRY)
    dt = kd.KD_BF16 if dtype == "bf16" else kd.KD_F32
    bws = torch.empty(kd.workspace_size(kd.KD_WS_BWD, 1, 3, 200, d, d, dt), dtype=torch.uint8, device="cuda")
    g2 = kd.bwd(*a, x["S0"], x["dO"], fwd_workspace=ws2, workspace=bws, phase=kd.KD_PHASE_LOCAL)
    g2 = kd.bwd(*a, x["S0"], x["dO"], fwd_workspace=ws2, workspace=bws, phase=kd.KD_PHASE_CARRY, grads=g2)
    torch.cuda.synchronize()
    kd.device_status()
    assert torch.equal(out1, out2) and torch.equal(ST1, ST2)
    for n in ("dq", "dk", "dv", "dbeta", "dc", "dlogf", "dS0"):
        assert torch.equal(g1[n], g2[n]), n


@pytest.mark.parametrize("dtype,d,bounds", [("bf16", 128, (0, 128, 320, 450)), ("f32", 64, (0, 100, 230))])
def test_segments_on_one_gpu_match_whole_sequence(oracle, dtype, d, bounds):
    T = bounds[-1]
    inp = kin.make_inputs(4, B=1, H=2, T=T, dk=d, dv=d, seed=11)
    dST = np.random.default_rng(2).standard_normal((1, 2, d, d)) / d
    segs = list(zip(bounds[:-1], bounds[1:]))
    xs = [dev(inp, dtype, lo, hi) for lo, hi in segs]
    dt = kd.KD_BF16 if dtype == "bf16" else kd.KD_F32
    # every segment's state-independent work first, as concurrent ranks would run it
    st = [kd.fwd(*(x[n] for n in ARGS), None, save=True, phase=kd.KD_PHASE_LOCAL) for x in xs]
    S_in, outs, S_ins = xs[0]["S0"], [], []
    for x, (out, ST, ws) in zip(xs, st):
        S_ins.append(S_in)
        out, ST, _ = kd.fwd(*(x[n] for n in ARGS), S_in, out=out, state_out=ST, save=True, workspace=ws,
                            phase=kd.KD_PHASE_CARRY)
        outs.append(out)
        S_in = ST.clone()  # the hand-off: the next segment's own copy
    bws = [torch.empty(kd.workspace_size(kd.KD_WS_BWD, 1, 2, hi - lo, d, d, dt), dtype=torch.uint8, device="cuda")
           for lo, hi in segs]
    gl = [kd.bwd(*(x[n] for n in ARGS), S, x["dO"], fwd_workspace=s[2], workspace=w, phase=kd.KD_PHASE_LOCAL)
          for x, S, s, w in zip(xs, S_ins, st, bws)]
    dS = torch.from_numpy(dST).float().cuda()
    grads = [None] * len(xs)
    for i in reversed(range(len(xs))):
        x = xs[i]
        grads[i] = kd.bwd(*(x[n] for n in ARGS), S_ins[i], x["dO"], dS, fwd_workspace=st[i][2], workspace=bws[i],
                          phase=kd.KD_PHASE_CARRY, grads=gl[i])
        dS = grads[i]["dS0"].clone()
    torch.cuda.synchronize()
    kd.device_status()
    O_ref, ST_ref = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["c"], inp["logf"], inp["S0"])
    g_ref = oracle.bwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["c"], inp["logf"], inp["S0"], inp["dO"], dST)
    tf, tg = TOL[dtype]
    assert rel(np.concatenate([host(o) for o in outs], axis=1), O_ref) <= tf
    assert rel(host(st[-1][1]), ST_ref) <= tf
    for n in ("dq", "dk", "dv", "dbeta", "dc", "dlogf"):
        e = rel(np.concatenate([host(g[n]) for g in grads], axis=1), g_ref[n])
        assert e <= tg, (n, e)
    assert rel(host(grads[0]["dS0"]), g_ref["dS0"]) <= tg


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime

    import torch.distributed as dist

    from delta_rule_linear_kron_b200 import relay

    class HostHandOff(relay.CudaSegmentOps):
        """The CUDA segment operations, with the carried state passed through
        host memory (gloo moves CPU tensors only)."""

        def new_state(self, like, B, H, dv, dk):
            return torch.empty((B, H, dv, dk), dtype=torch.float32)

        def fwd_carry(self, inputs, S_in, st):
            out, ST = super().fwd_carry(inputs, None if S_in is None else S_in.cuda(), st)
            return out, ST.cpu()

        def bwd_carry(self, inputs, S_in, st, dO, dST, bst):
            g = super().bwd_carry(inputs, S_in, st, dO, None if dST is None else dST.cuda(), bst)
            g["dS0"] = g["dS0"].cpu()
            return g

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(0)
    inp = kin.make_inputs(4, B=1, H=2, T=300, seed=21)
    lo, hi = (0, 140) if rank == 0 else (140, 300)
    x = dev(inp, "bf16", lo, hi)
    ops = HostHandOff()
    S0 = x["S0"]
    out, ST, ctx = relay.relay_fwd(*(x[n] for n in ARGS), S0, ops=ops)
    if rank == 0:
        ctx.S_in = S0
    else:
        ctx.S_in = ctx.S_in.cuda()
    g = relay.relay_bwd(ctx, x["dO"], None, ops=ops)
    torch.cuda.synchronize()
    kd.device_status()
    np.savez(os.path.join(out_dir, f"rank{rank}.npz"), out=host(out),
             ST=np.zeros(0) if ST is None else host(ST),
             **{n: host(g[n]) for n in ("dq", "dk", "dv", "dbeta", "dc", "dlogf", "dS0")})
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(dict(lo=lo, hi=hi), f)
    dist.destroy_process_group()


def test_relay_two_processes_through_host(tmp_path, oracle):
    import torch.multiprocessing as mp
    mp.start_processes(_rank_main, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    inp = kin.make_inputs(4, B=1, H=2, T=300, seed=21)
    O_ref, ST_ref = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["c"], inp["logf"], inp["S0"])
    g_ref = oracle.bwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["c"], inp["logf"], inp["S0"], inp["dO"], None)
    z = [np.load(tmp_path / f"rank{r}.npz") for r in range(2)]
    m = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    assert rel(np.concatenate([z[0]["out"], z[1]["out"]], axis=1), O_ref) <= 5e-3
    assert rel(z[1]["ST"], ST_ref) <= 5e-3
    for n in ("dq", "dk", "dv", "dbeta", "dc", "dlogf"):
        assert rel(np.concatenate([z[r][n] for r in range(2)], axis=1), g_ref[n]) <= 1e-2, n
    assert rel(z[0]["dS0"], g_ref["dS0"]) <= 1e-2
    assert m[0]["hi"] == m[1]["lo"]
