"""GPU parity of the output epilogue (kron_delta_epilogue_fwd / _bwd) against
the fp64 epilogue oracle on identical seeded inputs, element by element.

Tolerances, from the arithmetic (fp32 inside the kernel, one rounding to the
storage dtype on the way out): |x - ref| <= 2^-8 |ref| (bf16; 2^-22 for
fp32) plus 1e-5 of the row's largest magnitude for the fp32 row arithmetic
(a dv-term sum of squares, one rsqrt, a dv-term dot product, a few products).
dw is an fp32 sum over all rows in a fixed tree: within 1e-5 of the sum of
its terms' magnitudes.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import delta_rule_linear_kron_b200 as kd  # noqa: E402
from delta_rule_linear_kron_b200 import inputs as kin  # noqa: E402
from oracle import epilogue as E  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    kd.lib()


def dev(inp, dtype):
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    return {n: torch.from_numpy(x).to("cuda", dtype=torch.float32 if n == "w" else tdt).contiguous()
            for n, x in inp.items()}


def host(t):
    return t.detach().double().cpu().numpy()


def close_rows(x, ref, dtype, name):
    rel = 2.0 ** -8 if dtype == "bf16" else 2.0 ** -22
    slack = 1e-5 * np.max(np.abs(ref), axis=-1, keepdims=True) + 1e-30
    bad = np.abs(x - ref) > rel * np.abs(ref) + slack
    assert not bad.any(), f"{name}: {int(bad.sum())} elements off, first at {np.argwhere(bad)[0]}"


def run(inp, dtype):
    d = dev(inp, dtype)
    y = kd.epilogue_fwd(d["o"], d["g"], d["w"])
    r = kd.epilogue_bwd(d["o"], d["g"], d["w"], d["dy"])
    torch.cuda.synchronize()
    return y, r


def check(inp, dtype):
    y, r = run(inp, dtype)
    close_rows(host(y), E.epilogue_fwd(inp["o"], inp["g"], inp["w"]), dtype, "y")
    ref = E.epilogue_bwd(inp["o"], inp["g"], inp["w"], inp["dy"])
    close_rows(host(r["dO"]), ref["do"], dtype, "dO")
    close_rows(host(r["dg"]), ref["dg"], dtype, "dg")
    n, _ = E.rms_normalise(inp["o"])
    mag = np.sum(np.abs(inp["dy"] * n * E.sigmoid(inp["g"])), axis=(0, 1, 2))
    assert np.all(np.abs(host(r["dw"]) - ref["dw"]) <= 1e-5 * mag + 1e-7)


@pytest.mark.parametrize("dv", [32, 64, 128])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_epilogue_small(dv, dtype):
    check(kin.make_epilogue_inputs(2, 3, 77, dv, dtype, seed=dv), dtype)


@pytest.mark.parametrize("T", [1, 65, 999])
def test_epilogue_ragged(T):
    check(kin.make_epilogue_inputs(1, 5, T, 128, "bf16", seed=T), "bf16")


def test_epilogue_edge_values():
    """Zero read-out rows (output zero, gradient dy*w*s/sqrt(eps)), saturated
    gates (+-40) and a tiny read-out scale where eps matters."""
    inp = kin.make_epilogue_inputs(1, 4, 40, 64, "f32", seed=3)
    inp["o"][0, 2, 1, :] = 0.0
    inp["o"][0, 3, 2, :] *= 1e-3
    inp["g"][0, 5, :, :] = 40.0
    inp["g"][0, 6, :, :] = -40.0
    check(inp, "f32")


def test_epilogue_workload_B1_H16_T16384():
    """The mixer's full-size read-out (B=1, H=16, T=16384, dv=128, bf16), every element."""
    check(kin.make_epilogue_inputs(1, 16, 16384, 128, "bf16", seed=3004), "bf16")


def test_epilogue_bwd_deterministic():
    inp = kin.make_epilogue_inputs(2, 8, 3000, 128, "bf16", seed=9)
    _, r1 = run(inp, "bf16")
    _, r2 = run(inp, "bf16")
    for n in r1:
        assert torch.equal(r1[n], r2[n]), n
