"""GPU checks of kron_delta_bwd_recompute, the backward that reruns the
forward's chunk-local work and chunk chain instead of reading a saved forward
workspace.  The chunk form of the KronLSTM digest ("무엇과 다른가": the
DeltaNet chunk-parallel form) makes the saved quantities a pure function of
the inputs, and every kernel on the path is deterministic, so the gradients
must equal those of fwd(save=True) + bwd bit for bit.  One case per path
(tensor cores: bf16, d = 128, ragged T; CUDA cores: fp32, d = 64), and the
tensor-core case also against the fp64 oracle.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import delta_rule_linear_kron_b200 as kd  # noqa: E402
from delta_rule_linear_kron_b200 import inputs as kin  # noqa: E402

GRADS = ("dq", "dk", "dv", "dbeta", "dc", "dlogf", "dS0")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    kd.lib()


def _run(inp, tdt, with_dST):
    d = {n: torch.from_numpy(inp[n]).to("cuda", tdt) for n in ("q", "k", "v", "dO")}
    for n in ("beta", "c", "logf"):
        d[n] = torch.from_numpy(inp[n]).to("cuda", torch.float32)
    d["S0"] = None if inp["S0"] is None else torch.from_numpy(inp["S0"]).to("cuda", torch.float32)
    B, T, H, dk = inp["q"].shape
    dv = inp["v"].shape[-1]
    dST = None
    if with_dST:
        dST = torch.from_numpy(np.random.default_rng(77).normal(size=(B, H, dv, dk))).to("cuda", torch.float32)
    args = (d["q"], d["k"], d["v"], d["beta"], d["c"], d["logf"], d["S0"])
    _, _, ws = kd.fwd(*args, save=True)
    saved = kd.bwd(*args, d["dO"], dST, fwd_workspace=ws)
    rec = kd.bwd(*args, d["dO"], dST, fwd_workspace=None)
    torch.cuda.synchronize()
    kd.device_status()
    return saved, rec


@pytest.mark.parametrize("case", [
    dict(wl=4, B=2, H=3, T=1000, d=128, dST=True),   # bf16, tensor cores, nonzero S0, ragged tail
    dict(wl=1, B=1, H=2, T=300, d=64, dST=False),    # fp32, CUDA cores, S0 = 0
])
def test_recompute_equals_saved_forward(case):
    inp = kin.make_inputs(case["wl"], B=case["B"], H=case["H"], T=case["T"], dk=case["d"], dv=case["d"], seed=4242)
    tdt = torch.bfloat16 if kin.WORKLOADS[case["wl"]].dtype == "bf16" else torch.float32
    saved, rec = _run(inp, tdt, case["dST"])
    for n in GRADS:
        if saved[n] is not None:
            assert torch.equal(saved[n], rec[n]), n


def test_recompute_matches_the_oracle(oracle):
    inp = kin.make_inputs(4, B=1, H=2, T=700, seed=4243)
    _, rec = _run(inp, torch.bfloat16, False)
    gr = oracle.bwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["c"], inp["logf"], inp["S0"], inp["dO"], None)
    for n in GRADS:
        x = rec[n].double().cpu().numpy()
        err = np.linalg.norm(x - gr[n]) / max(np.linalg.norm(gr[n]), 1e-300)
        assert err < 1e-2, (n, err)
