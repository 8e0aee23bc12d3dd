"""Runs the forward+backward step of the Kronecker delta rule mixer at a
chosen shape, for profilers (ncu) that need a small, repeatable case.

    python -m delta_rule_linear_kron_b200.profile_step [--B 1] [--H 16] [--T 2048] [--steps 4]

Inputs follow the forward+backward workload's recipe (bf16 q, k, v, dO; fp32
gates; beta in (0, 2); nonzero S0) at the given shape.  Each step is one
forward (saving for the backward) and one backward, as in bench.py.
"""
from __future__ import annotations

import argparse
import sys


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--B", type=int, default=1)
    ap.add_argument("--H", type=int, default=16)
    ap.add_argument("--T", type=int, default=2048)
    ap.add_argument("--steps", type=int, default=4)
    a = ap.parse_args(argv)

    import torch

    import delta_rule_linear_kron_b200 as kd
    from delta_rule_linear_kron_b200 import inputs as kin

    inp = kin.make_inputs(4, B=a.B, H=a.H, T=a.T)
    d = {n: torch.from_numpy(inp[n]).to("cuda", torch.bfloat16 if n in ("q", "k", "v", "dO") else torch.float32)
         for n in ("q", "k", "v", "dO", "beta", "c", "logf", "S0")}
    fws = torch.empty(kd.workspace_size(kd.KD_WS_FWD_SAVE, a.B, a.H, a.T, 128, 128), dtype=torch.uint8,
                      device="cuda")
    bws = torch.empty(kd.workspace_size(kd.KD_WS_BWD, a.B, a.H, a.T, 128, 128), dtype=torch.uint8, device="cuda")
    for _ in range(a.steps):
        kd.fwd(d["q"], d["k"], d["v"], d["beta"], d["c"], d["logf"], d["S0"], save=True, workspace=fws)
        kd.bwd(d["q"], d["k"], d["v"], d["beta"], d["c"], d["logf"], d["S0"], d["dO"], fwd_workspace=fws,
               workspace=bws)
    torch.cuda.synchronize()
    kd.device_status()
    print(f"profile_step: {a.steps} fwd+bwd steps at B={a.B} H={a.H} T={a.T} done")
    return 0


if __name__ == "__main__":
    sys.exit(main())
