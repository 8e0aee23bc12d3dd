"""Runs the forward+backward step of the Kronecker delta rule mixer at a
chosen shape, for profilers (ncu) that need a small, repeatable case.

    python -m delta_rule_linear_kron_b200.profile_step [--B 1] [--H 16] [--T 2048] [--steps 4] [--gated | --gdn2]

Inputs follow the forward+backward workload's recipe (bf16 q, k, v, dO; fp32
gates; beta in (0, 2); nonzero S0) at the given shape.  Each step is one
forward (saving for the backward) and one backward, as in bench.py.  With
--gated the step goes through the gated entry points instead, with the forget
gate as a bf16 pre-activation ~ N(3, 1) and a_log ~ U(-1, 1).  With --gdn2 each
step is the Gated DeltaNet-2 rule's forward and backward at the same shape
(unit-norm bf16 q, k, v; sigmoid gates b, w; log-decays -softplus(N(0,1) - 4)).
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
    ap.add_argument("--gated", action="store_true")
    ap.add_argument("--gdn2", action="store_true")
    a = ap.parse_args(argv)

    import torch

    import delta_rule_linear_kron_b200 as kd
    from delta_rule_linear_kron_b200 import inputs as kin

    if a.gdn2:
        return gdn2_steps(a, torch, kd)
    inp = kin.make_inputs(4, B=a.B, H=a.H, T=a.T)
    d = {n: torch.from_numpy(inp[n]).to("cuda", torch.bfloat16 if n in ("q", "k", "v", "dO") else torch.float32)
         for n in ("q", "k", "v", "dO", "beta", "c", "logf", "S0")}
    kf, kb = (kd.KD_WS_FWD_GATED, kd.KD_WS_BWD_GATED) if a.gated else (kd.KD_WS_FWD_SAVE, kd.KD_WS_BWD)
    fws = torch.empty(kd.workspace_size(kf, a.B, a.H, a.T, 128, 128), dtype=torch.uint8, device="cuda")
    bws = torch.empty(kd.workspace_size(kb, a.B, a.H, a.T, 128, 128), dtype=torch.uint8, device="cuda")
    if a.gated:
        g = torch.Generator(device="cuda")
        g.manual_seed(3004)
        f_pre = (torch.randn(d["logf"].shape, generator=g, device="cuda") + 3.0).to(torch.bfloat16)
        a_log = torch.rand((a.H,), generator=g, device="cuda") * 2 - 1
    for _ in range(a.steps):
        if a.gated:
            kd.fwd_gated(d["q"], d["k"], d["v"], d["beta"], d["c"], f_pre, a_log, d["S0"], save=True, workspace=fws)
            kd.bwd_gated(d["q"], d["k"], d["v"], d["beta"], d["c"], f_pre, a_log, d["S0"], d["dO"],
                         fwd_workspace=fws, workspace=bws)
        else:
            kd.fwd(d["q"], d["k"], d["v"], d["beta"], d["c"], d["logf"], d["S0"], save=True, workspace=fws)
            kd.bwd(d["q"], d["k"], d["v"], d["beta"], d["c"], d["logf"], d["S0"], d["dO"], fwd_workspace=fws,
                   workspace=bws)
    torch.cuda.synchronize()
    kd.device_status()
    print(f"profile_step: {a.steps} {'gated ' if a.gated else ''}fwd+bwd steps at B={a.B} H={a.H} T={a.T} done")
    return 0


def gdn2_steps(a, torch, kd):
    g = torch.Generator(device="cuda")
    g.manual_seed(4004)
    B, H, T, d = a.B, a.H, a.T, 128

    def unit(*sh):
        x = torch.randn(sh, generator=g, device="cuda")
        return (x / x.norm(dim=-1, keepdim=True)).to(torch.bfloat16)
    q, k, v = unit(B, T, H, d), unit(B, T, H, d), unit(B, T, H, d)
    b = torch.sigmoid(torch.randn((B, T, H, d), generator=g, device="cuda"))
    w = torch.sigmoid(torch.randn((B, T, H, d), generator=g, device="cuda"))
    la = -torch.nn.functional.softplus(torch.randn((B, T, H, d), generator=g, device="cuda") - 4.0)
    dO = torch.randn((B, T, H, d), generator=g, device="cuda").to(torch.bfloat16)
    S0 = torch.randn((B, H, d, d), generator=g, device="cuda") / d
    fws = torch.empty(kd.workspace_size(kd.KD_WS_GDN2_FWD, B, H, T, d, d), dtype=torch.uint8, device="cuda")
    bws = torch.empty(kd.workspace_size(kd.KD_WS_GDN2_BWD, B, H, T, d, d), dtype=torch.uint8, device="cuda")
    for _ in range(a.steps):
        kd.gdn2_fwd(q, k, v, b, w, la, S0, workspace=fws)
        kd.gdn2_bwd(q, k, v, b, w, la, S0, dO, fwd_workspace=fws, workspace=bws)
    torch.cuda.synchronize()
    kd.device_status()
    print(f"profile_step: {a.steps} Gated DeltaNet-2 fwd+bwd steps at B={B} H={H} T={T} done")
    return 0


if __name__ == "__main__":
    sys.exit(main())
