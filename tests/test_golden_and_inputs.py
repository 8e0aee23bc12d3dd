"""Hand-worked golden example for the oracle, and checks of the seeded input
generator (dtype rounding, shapes, distributions)."""
import os

import numpy as np
import torch

from delta_rule_linear_kron_b200 import inputs as kin

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked_2x2_T3.txt")


def _read_golden():
    rows, S3 = [], None
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line.startswith("S3"):
            S3 = np.array([float(x) for x in line.split()[1:]]).reshape(2, 2)
            continue
        lhs, rhs = line.split("|")
        rows.append(([float(x) for x in lhs.split()], [float(x) for x in rhs.split()]))
    return rows, S3


def test_hand_worked_example(oracle):
    rows, S3 = _read_golden()
    T = len(rows)
    q = np.zeros((1, T, 1, 2)); k = np.zeros_like(q); v = np.zeros_like(q)
    beta = np.zeros((1, T, 1)); c = np.zeros_like(beta); logf = np.zeros_like(q)
    for t, (x, _) in enumerate(rows):
        k[0, t, 0] = x[1:3]; v[0, t, 0] = x[3:5]; q[0, t, 0] = x[5:7]
        beta[0, t, 0] = x[7]; c[0, t, 0] = x[8]; logf[0, t, 0] = np.log(x[9:11])
    O, ST, bt, ut = oracle.fwd(q, k, v, beta, c, logf, None, want_bu=True)
    for t, (_, y) in enumerate(rows):
        assert np.allclose(O[0, t, 0], y[0:2], atol=1e-12)
        assert abs(bt[0, t, 0] - y[2]) < 1e-12 and abs(ut[0, t, 0] - y[3]) < 1e-12
    assert np.allclose(ST[0, 0], S3, atol=1e-12)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000), rng.standard_normal(1000) * 1e-30,
                        rng.standard_normal(1000) * 1e30, [0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8]])
    mine = kin.round_to_dtype(x, "bf16")
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).double().numpy()
    assert np.array_equal(mine, ref)


def test_workload_inputs_shapes_and_ranges():
    inp = kin.make_inputs(1)
    wl = inp["wl"]
    assert inp["q"].shape == (wl.B, wl.T, wl.H, wl.dk) and inp["v"].shape == (wl.B, wl.T, wl.H, wl.dv)
    assert np.allclose(np.linalg.norm(inp["k"], axis=-1), 1.0, atol=1e-6)
    assert np.all((inp["beta"] > 0) & (inp["beta"] < 1)) and np.all((inp["c"] > 0) & (inp["c"] < 1))
    assert np.all(inp["logf"] < 0) and inp["S0"] is None
    small = kin.make_inputs(4, T=200, H=3)
    assert np.all(small["beta"] < 2) and small["beta"].max() > 1
    assert np.allclose(np.linalg.norm(small["S0"], axis=(-2, -1)), 1.0, atol=1e-6)
    # bf16 storage: every q value is bf16-representable
    assert np.array_equal(kin.round_to_dtype(small["q"], "bf16"), small["q"])
    # a_h is per head: the ratio of mean logf between heads varies, within a head it does not
    again = kin.make_inputs(4, T=200, H=3)
    assert np.array_equal(again["logf"], small["logf"])
    d = kin.make_decode_inputs(2, B=3, H=2)
    assert d["S"].shape == (3, 2, 128, 128) and abs(d["S"].std() - 128 ** -0.5) < 0.01
