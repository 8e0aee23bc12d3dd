"""Context-parallel relay (delta_rule_linear_kron_b200.relay), host logic on
CPU: 2 and 3 gloo ranks, each holding one time segment of every sequence, with
the segment operations done by the fp64 oracle (test infrastructure; the
package's own segment operations are the CUDA kernels, checked on the GPU in
test_gpu_relay.py).  The relayed forward and backward must equal the oracle on
the whole sequence: outputs, final state, every input gradient and dS0."""
import json
import os
import socket

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleSegmentOps:
    """The relay's segment operations done by the fp64 oracle, on torch CPU tensors."""

    def __init__(self, oracle):
        self.o = oracle

    def new_state(self, like, B, H, dv, dk):
        import torch
        return torch.empty((B, H, dv, dk), dtype=torch.float64)

    def fwd_local(self, inputs, save):
        return {}

    def fwd_carry(self, inputs, S_in, st):
        import torch
        out, ST = self.o.fwd(*(x.numpy() for x in inputs), None if S_in is None else S_in.numpy())
        return torch.from_numpy(out), torch.from_numpy(ST)

    def bwd_local(self, inputs, S_in, st, dO):
        return {}

    def bwd_carry(self, inputs, S_in, st, dO, dST, bst):
        import torch
        g = self.o.bwd(*(x.numpy() for x in inputs), None if S_in is None else S_in.numpy(), dO.numpy(),
                       None if dST is None else dST.numpy())
        return {n: torch.from_numpy(x) for n, x in g.items()}


def _problem(T):
    from delta_rule_linear_kron_b200 import inputs as kin
    inp = kin.make_inputs(4, B=2, H=2, T=T, dk=16, dv=8, seed=77)
    dST = np.random.default_rng(3).standard_normal((2, 2, 8, 16))
    return inp, dST


def _rank_main(rank, world, port, T, out_dir):
    import datetime

    import torch
    import torch.distributed as dist

    from delta_rule_linear_kron_b200 import relay
    from oracle import oracle as O
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    inp, dST = _problem(T)
    seg = T // world
    lo, hi = rank * seg, (rank + 1) * seg if rank < world - 1 else T
    x = {n: torch.from_numpy(np.ascontiguousarray(inp[n][:, lo:hi])) for n in ("q", "k", "v", "beta", "c", "logf",
                                                                              "dO")}
    ops = OracleSegmentOps(O)
    out, ST, ctx = relay.relay_fwd(x["q"], x["k"], x["v"], x["beta"], x["c"], x["logf"],
                                   torch.from_numpy(inp["S0"]), ops=ops)
    g = relay.relay_bwd(ctx, x["dO"], torch.from_numpy(dST), ops=ops)
    np.savez(os.path.join(out_dir, f"rank{rank}.npz"), out=out.numpy(), ST=np.zeros(0) if ST is None else ST.numpy(),
             **{n: g[n].numpy() for n in ("dq", "dk", "dv", "dbeta", "dc", "dlogf", "dS0")})
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(dict(lo=lo, hi=hi, has_ST=ST is not None), f)
    dist.destroy_process_group()


@pytest.mark.parametrize("world,T", [(2, 192), (3, 200)])
def test_relay_matches_whole_sequence(tmp_path, oracle, world, T):
    import torch.multiprocessing as mp
    mp.start_processes(_rank_main, args=(world, _free_port(), T, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    inp, dST = _problem(T)
    O_ref, ST_ref = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["c"], inp["logf"], inp["S0"])
    g_ref = oracle.bwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["c"], inp["logf"], inp["S0"], inp["dO"], dST)
    for r in range(world):
        meta = json.load(open(tmp_path / f"rank{r}.json"))
        z = np.load(tmp_path / f"rank{r}.npz")
        lo, hi = meta["lo"], meta["hi"]
        assert np.allclose(z["out"], O_ref[:, lo:hi], rtol=1e-11, atol=1e-12)
        assert meta["has_ST"] == (r == world - 1)
        if r == world - 1:
            assert np.allclose(z["ST"], ST_ref, rtol=1e-11, atol=1e-12)
        for n in ("dq", "dk", "dv", "dbeta", "dc", "dlogf"):
            assert np.allclose(z[n], g_ref[n][:, lo:hi], rtol=1e-10, atol=1e-11), (r, n)
        if r == 0:
            assert np.allclose(z["dS0"], g_ref["dS0"], rtol=1e-10, atol=1e-11)
