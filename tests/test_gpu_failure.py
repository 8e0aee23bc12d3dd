"""Failure reporting on the GPU without faulting it: a bounded device-side
wait that is made to run out (a barrier nothing arrives at) must surface as
KD_ERR_TIMEOUT from kron_delta_device_status, clear itself, and leave the
context usable for the next call."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import delta_rule_linear_kron_b200 as kd  # noqa: E402
from delta_rule_linear_kron_b200 import inputs as kin  # noqa: E402


def test_bounded_wait_timeout_is_reported_and_cleared(oracle):
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    torch.cuda.synchronize()
    kd.device_status()  # nothing pending
    stream = torch.cuda.current_stream()
    assert kd.lib().kron_delta_selftest_timeout(kd._stream(None)) == kd.KD_OK
    with pytest.raises(kd.KronDeltaError) as ei:
        kd.device_status()
    assert ei.value.code == kd.KD_ERR_TIMEOUT
    kd.device_status()  # cleared by the previous report
    # the context still works: a small forward matches the oracle
    inp = kin.make_inputs(1, B=1, H=2, T=70, seed=3)
    d = {n: torch.from_numpy(inp[n]).float().cuda() for n in ("q", "k", "v", "beta", "c", "logf")}
    out, ST, _ = kd.fwd(d["q"], d["k"], d["v"], d["beta"], d["c"], d["logf"])
    stream.synchronize()
    kd.device_status()
    O_ref, _ = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["c"], inp["logf"], None)
    x = out.double().cpu().numpy()
    assert np.linalg.norm(x - O_ref) <= 1e-4 * np.linalg.norm(O_ref)
