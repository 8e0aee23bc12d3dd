"""Pins of the epilogue oracle (oracle/epilogue.py): a closed form, torch's
own RMSNorm and sigmoid in float64 on the CPU (an independent library
routine), central finite differences for the backward, and planted mistakes
that the pins must reject.  CPU only."""
import numpy as np
import pytest
import torch

from oracle import epilogue as _E


def _inputs(seed, B=2, T=5, H=3, dv=8):
    r = np.random.default_rng(seed)
    return dict(o=r.normal(size=(B, T, H, dv)) * 0.3, g=r.normal(size=(B, T, H, dv)) * 2,
                w=r.normal(size=(dv,)) * 0.5 + 1.0)


def test_constant_row_closed_form(E=_E):
    o = np.full((1, 1, 1, 4), -2.0)
    g = np.zeros((1, 1, 1, 4))
    w = np.array([1.0, 2.0, 3.0, 4.0])
    y = E.epilogue_fwd(o, g, w, eps=0.0)
    # mean(o^2) = 4, so o / rms = -1; sigmoid(0) = 1/2
    assert np.allclose(y.reshape(-1), -0.5 * w, rtol=1e-15)
    y = E.epilogue_fwd(o, g, w)
    assert np.allclose(y.reshape(-1), -0.5 * w * 2.0 / np.sqrt(4.0 + 1e-6), rtol=1e-15)
    # a zero read-out stays zero
    assert np.all(E.epilogue_fwd(np.zeros((1, 1, 1, 4)), g, w) == 0)


def test_forward_matches_torch_rms_norm(E=_E):
    x = _inputs(1)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x["o"]), (8,), weight=torch.from_numpy(x["w"]), eps=1e-6)
    ref = (ref * torch.sigmoid(torch.from_numpy(x["g"]))).numpy()
    assert np.allclose(E.epilogue_fwd(**x), ref, rtol=1e-13, atol=1e-15)


def test_backward_matches_torch_autograd(E=_E):
    x = _inputs(2)
    dy = np.random.default_rng(3).normal(size=x["o"].shape)
    t = {n: torch.from_numpy(v.copy()).requires_grad_(True) for n, v in x.items()}
    y = torch.nn.functional.rms_norm(t["o"], (8,), weight=t["w"], eps=1e-6) * torch.sigmoid(t["g"])
    (y * torch.from_numpy(dy)).sum().backward()
    g = E.epilogue_bwd(**x, dy=dy)
    for n in ("o", "g", "w"):
        assert np.allclose(g["d" + n], t[n].grad.numpy(), rtol=1e-11, atol=1e-13), n


def test_backward_matches_central_differences(E=_E):
    x = _inputs(4, B=1, T=3, H=2, dv=4)
    dy = np.random.default_rng(5).normal(size=x["o"].shape)
    g = E.epilogue_bwd(**x, dy=dy)
    h = 1e-6
    for n in ("o", "g", "w"):
        flat = x[n].reshape(-1)
        fd = np.zeros(flat.size)
        for i in range(flat.size):
            keep = flat[i]
            flat[i] = keep + h
            lp = float(np.sum(dy * E.epilogue_fwd(**x)))
            flat[i] = keep - h
            lm = float(np.sum(dy * E.epilogue_fwd(**x)))
            flat[i] = keep
            fd[i] = (lp - lm) / (2 * h)
        assert np.allclose(g["d" + n].reshape(-1), fd, rtol=1e-6, atol=1e-8), n


MUTANTS = [
    ("sum-not-mean", "np.mean(o * o, axis=-1, keepdims=True) + eps", "np.sum(o * o, axis=-1, keepdims=True) + eps"),
    ("no-sqrt", "r = 1.0 / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps)",
     "r = 1.0 / (np.mean(o * o, axis=-1, keepdims=True) + eps)"),
    ("no-eps", "keepdims=True) + eps)", "keepdims=True))"),
    ("no-weight", "return _f64(w) * n * sigmoid(g)", "return n * sigmoid(g)"),
    ("do-no-projection", "do = r * (dn - n * np.mean(n * dn, axis=-1, keepdims=True))", "do = r * dn"),
    ("do-sum-not-mean", "n * np.mean(n * dn, axis=-1", "n * np.sum(n * dn, axis=-1"),
    ("dg-no-complement", "dg = dy * w * n * s * sigmoid(-g)", "dg = dy * w * n * s"),
    ("dw-no-gate", "dw = np.sum(dy * n * s,", "dw = np.sum(dy * n,"),
    ("dn-no-gate", "dn = dy * w * s", "dn = dy * w"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_reject_mutant(tmp_path, name, old, new):
    import importlib.util
    src = open(_E.__file__).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    f = tmp_path / f"epilogue_{name.replace('-', '_')}.py"
    f.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location(f.stem, f)
    M = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(M)
    caught = 0
    for pin in (test_constant_row_closed_form, test_forward_matches_torch_rms_norm,
                test_backward_matches_torch_autograd, test_backward_matches_central_differences):
        try:
            pin(M)
        except AssertionError:
            caught += 1
    assert caught > 0, f"no pin rejects mutant {name}"
