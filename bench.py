#!/usr/bin/env python3
"""Benchmark of the Kronecker delta rule mixer on B200.

One step = one pass of the whole hot path over one batch: the chunked
forward (saving what the backward needs) followed by the backward, on the
forward+backward workload B=1, H=16, T=16384, d_k=d_v=128, bf16 q/k/v/dO,
fp32 gates and state, beta in (0,2), nonzero S0.  The decode step
(B=256, H=16, d=128, 1000 consecutive in-place steps) is timed in the same run
and reported under "decode"; the input prologue (raw projections -> normalised
q, k, v and gates), the output epilogue (RMSNorm and output gate) and their
backward passes, on the step's shape, under "prologue_epilogue"; the Gated
DeltaNet-2 rule's forward + backward on the same shape under "gdn2".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (launched by torchrun): each rank runs its own batch of the same
shape (independent (b,h) units, no collective on the data path; weak
scaling); time is the max over ranks.  Inputs (~0.5 GB per step) are larger
than L2 (126 MB), so no L2 flush is needed between steps.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WL = dict(B=1, H=16, T=16384, dk=128, dv=128)
CHUNK = 64
METRIC = "Kron-delta fwd+bwd tokens/s (H16,d128,T16K) & % bf16 TC peak; decode GB/s"
WORKLOAD_NAME = "fwdbwd-B1-H16-T16384-d128-beta2"
REF_STEP_T = 512        # tokens per step of the reference (oracle) arm


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm_gbs=d["hbm_gbs"], bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                    sm_max_mhz=d.get("sm_max_mhz", 1965.0), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, sm_max_mhz=1965.0,
                source="fallback")


# ---------------------------------------------------------------------------
# Algorithmic work, per token-head (d_k = d_v = d = 128, C = 64, bf16
# activations, fp32 gates).  The method's rows and their dense contractions
# (2 flops per multiply-add; C x C tiles counted whole, the O(C^3) solve and
# elementwise work not counted):
#   a2 Hadamard Gram       2 C x C x d   32,768     a3 query-key decay P   C x C x d   16,384
#   a5 chain erase read    d x d x C     32,768     a7 chain state update  d x d x C   32,768
#   a8 output              d x d x C + C x C x d                                       49,152
#   a9 reverse chain       3 d x d x C                                                 98,304
#   a10 backward intra     4 d x d x C + 8 C x C x d                                  262,144
# forward 163,840, backward 360,448, step 524,288.  Bytes: only what the
# operation must move (no intermediates): forward reads q, k, v (768 B),
# beta, c (8 B), logf (512 B) and writes O (256 B) = 1,544 B; the backward
# reads the same plus dO and writes dq, dk, dv, dbeta, dc, dlogf = 2,832 B;
# step 4,376 B.  Per-head states (S0, S_T, dS0: 64 KB each) are added exactly.
# ---------------------------------------------------------------------------
STEP_FLOPS = 524288
STEP_BYTES = 4376
FWD_FLOPS = 163840
FWD_BYTES = 1544


def method_work(name, d=128, C=CHUNK):
    """The method rows a kernel of the step executes, their flops per
    token-head, and the bytes of the method's own inputs it must read and
    outputs it must write (its share of the step's 4,376 B; workspace
    intermediates are not counted).  Kernels that only prepare lookahead
    operands carry no method flops."""
    act, lf, gate = d * 2, d * 4, 4
    dd, cd = 2 * d * d, 2 * C * d
    table = {
        # a1-a4: decay prefix, Grams, P, the chunk inverse (reads q, k, v, beta, c, logf)
        "fwd_prep_tc": ("a1-a4", 2 * cd + cd, 3 * act + 2 * gate + lf),
        # chain operands and the lookahead's cross-chunk matrix (reads k, v, logf)
        "fwd_cross_tc": ("lookahead operands", 0, 2 * act + lf),
        # a5-a7 (reads beta; S0 in, S_T out per head)
        "fwd_chain_tc": ("a5-a7", 2 * dd, gate),
        # a8 (reads q, k, v, logf; writes O)
        "fwd_out_tc": ("a8", dd + cd, 3 * act + lf + act),
        # a10, the part known before the chain (reads k, v, dO, logf)
        "bwd_pre_tc": ("a10 (pre-chain)", 0, 3 * act + lf),
        # a9 (reads beta; dS_T in, dS0 out per head)
        "bwd_chain_tc": ("a9", 3 * dd, gate),
        # a10 (reads q, k, v, dO, logf, beta, c; writes dq, dk, dv, dbeta, dc, dlogf)
        "bwd_post_tc": ("a10", 4 * dd + 8 * cd, 4 * act + lf + 2 * gate + 3 * act + 2 * gate + lf),
    }
    w = table.get(name)
    return None if w is None else dict(rows=w[0], flops=w[1], bytes=w[2])


# The bytes each kernel of the step actually moves by design, per token-head:
# its method inputs and outputs plus the workspace intermediates it writes and
# reads (for the traffic comparison with ncu's DRAM counters).  The
# cross-chunk kernel's tiles of the previous chunk, read just before by that
# chunk's own CTA and found in L2, are not counted.
def kernel_io_bytes(name, d=128, C=CHUNK):
    act = d * 2                      # one bf16 activation row
    lf = d * 4                       # one fp32 row (logf, K~, K^e, K+)
    tile_bf16 = d * d * 2 // C       # one bf16 d x d tile per chunk, per token
    cc = C * 4                       # one fp32 C x C matrix per chunk, per token
    ccb = C * 2                      # one bf16 C x C tile per chunk, per token
    vt = d * C * 2 // C              # one bf16 d x C tile per chunk (V^T, Q+^T), per token
    table = {
        # q, k, v, logf, beta, c in; y, A, P out
        "fwd_prep_tc": 3 * act + lf + 8 + 4 + 2 * cc,
        # v, k, logf in; K~, K^e, gamma_C, H, V^T out
        "fwd_cross_tc": 2 * act + lf + 2 * lf + 8 + cc + vt,
        # K~, K^e, V^T, A, H, y, beta, gamma_C in; u, b0, the bf16 chunk-start state out
        "fwd_chain_tc": 2 * lf + vt + 2 * cc + 4 + 4 + 8 + 8 + tile_bf16,
        # q, k, v, logf, u, chunk-start state in; O out
        "fwd_out_tc": 3 * act + lf + 4 + tile_bf16 + act,
        # v, dO, k, q, logf, P, u in; du, M u, [dP; E_V], P diag(u), E_K, K+, Q+^T out
        "bwd_pre_tc": 4 * act + lf + cc + 4 + 8 + 2 * ccb + ccb + ccb + lf + vt,
        # dO, K^e, K+, beta, A, H, gamma_C, V^T, Q+^T, du in; dS tile, g out
        "bwd_chain_tc": act + 2 * lf + 4 + 2 * cc + 8 + 2 * vt + 4 + tile_bf16 + 4,
        # logf, q, k, E_K, S0, dS, dO, v, [dP; E_V], P diag(u), u, b0, g, M u, beta in;
        # dq, dk, dv, dlogf, dbeta, dc out
        "bwd_post_tc": lf + 2 * act + ccb + 2 * tile_bf16 + 2 * act + 2 * ccb + ccb + 16 + 4 + 3 * act + lf + 8,
    }
    return table.get(name)


# The standalone prologue / epilogue passes (timed on their own): bytes per
# token-head of their own inputs and outputs; they are row-wise and HBM-bound.
def pass_bytes(name, d=128):
    act, lf = d * 2, d * 4
    return {
        "prologue_fwd": 4 * act + 8 + 3 * act + lf + 8,
        "prologue_bwd": 4 * act + 3 * act + lf + 16 + 4 * act + 8,
        "epilogue_fwd": 2 * act + act,
        "epilogue_bwd": 3 * act + 2 * act,
    }.get(name)


# DRAM bytes (read + write) per launch from one ncu capture of this workload
# (dram__bytes_read.sum + dram__bytes_write.sum), with the source file the
# kernel lives in and the first 16 hex digits of its sha256 at capture time;
# a kernel whose source has changed since reports no traffic.
NCU_TRAFFIC = {
    "fwd_prep_tc": (447285931, "kd_fwd_tc.cu", "0ec6969ffa6a3978"),
    "fwd_cross_tc": (619036160, "kd_fwd_tc.cu", "0ec6969ffa6a3978"),
    "fwd_chain_tc": (591101867, "kd_fchain_tc.cu", "cac9ee1a46a36d26"),
    "fwd_out_tc": (525770240, "kd_fwd_tc.cu", "0ec6969ffa6a3978"),
    "bwd_pre_tc": (768061696, "kd_bwd_chunk_tc.cu", "7c3d2764ee32d35f"),
    "bwd_chain_tc": (727406592, "kd_bchain_tc.cu", "b514c715eaf3ed73"),
    "bwd_post_tc": (1127274325, "kd_bwd_chunk_tc.cu", "7c3d2764ee32d35f"),
}


def ncu_traffic(name):
    t = NCU_TRAFFIC.get(name)
    if t is None:
        return None
    import hashlib
    path = os.path.join(ROOT, "delta_rule_linear_kron_b200", "csrc", t[1])
    try:
        with open(path, "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()[:16]
    except OSError:
        return None
    return t[0] if digest == t[2] else None


def fp32_alu_peak_tflops(sm_mhz):
    return 148 * 128 * 2 * sm_mhz * 1e6 / 1e12


# ---------------------------------------------------------------------------
# Gated DeltaNet-2 kernels: algorithmic flops per token-head at d_k = d_v = d,
# C = 64, counting each dense product of the chunk form once (full C x C tiles,
# as for the Kronecker kernels; exponentials and the O(C^3) inverse not
# counted).  The "_tc" kernels (bf16, d = 128) run their products on tcgen05
# and are held against the bf16 tensor peak; the others run on fp32 CUDA cores.
# ---------------------------------------------------------------------------
def gdn2_kernel_flops(name, d=128, C=CHUNK):
    dd, cd = 2 * d * d, 2 * C * d
    table = {
        "gdn2_prep": 2 * cd + 2 * cd,           # T, P; W = A E+, U' = A Z
        "gdn2_chain": 2 * dd,                   # U = U' - W S0^T; S <- S Gamma + U^T K^e
        "gdn2_out": dd + cd,                    # Q+ S0^T + P U
        "gdn2_bchain": cd + 3 * dd,             # P^T dO, K^e dS^T; dO^T Q+, dU^T W
        "gdn2_bpost_a": 3 * dd + 5 * cd,        # dQ+, dK^e, dW; dP, dZ, dE; dT (two products)
        "gdn2_bpost_b": 4 * cd,                 # dT K-, dP K-, dT^T E+, dP^T Q+
        "gdn2_prep_tc": 2 * cd + 2 * cd,
        "gdn2_chain_tc": 2 * dd,
        "gdn2_out_tc": dd + cd,
        "gdn2_bpre_tc": cd + dd,                # P^T dO; dO^T Q+
        "gdn2_bchain_tc": 2 * dd,               # K^e dS^T; dU^T W
        "gdn2_bpost_tc": 3 * dd + 9 * cd,       # the products of bpost_a and bpost_b
    }
    return table.get(name)


# ---------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi clock/throttle samples every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=["nvidia-smi unavailable"], samples=0)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return dict(sm_mhz=statistics.median(sm) if sm else None, sm_max_mhz=max(mx) if mx else None,
                    reasons=reasons, samples=len(rows))


# ---------------------------------------------------------------------------
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(x, world_size, device):
    """The job's time is the slowest rank's: all-reduce MAX of a float (any
    backend; the tensor lives on `device`)."""
    if world_size == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world_size, units_per_rank, steps, ms_total):
    """Whole-job rate under weak scaling: every rank processes units_per_rank
    per step (its own batch), and the job takes the slowest rank's time."""
    return world_size * units_per_rank * steps / (ms_total / 1e3)


def rank_seed(base, rank):
    """Each rank draws its own batch of the same shape."""
    return base + rank


def _oracle_time(inp, nthreads, bwd=True):
    from oracle import oracle
    t = time.perf_counter()
    oracle.fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["c"], inp["logf"], inp["S0"], nthreads=nthreads)
    if bwd:
        oracle.bwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["c"], inp["logf"], inp["S0"], inp["dO"],
                   nthreads=nthreads)
    return time.perf_counter() - t


def oracle_baseline(T1=1024, full=False, seed=1004):
    """The fp64 oracle, as it stands, on the host cores: the whole forward +
    backward workload threaded over its heads, and its first T1 tokens of
    every head on one thread.  full=True adds the whole workload on one thread
    and the long-context forward workload (B1 H16 T16384, forward only) both
    ways, a few minutes of CPU time."""
    from delta_rule_linear_kron_b200 import inputs as kin
    cores = len(os.sched_getaffinity(0))
    used = min(cores, WL["H"])
    inp = kin.make_inputs(4, seed=seed)
    el = _oracle_time(inp, cores)
    one = {n: inp[n][:, :T1] for n in ("q", "k", "v", "beta", "c", "logf", "dO")}
    one["S0"] = inp["S0"]
    el1 = _oracle_time(one, 1)
    out = dict(value=WL["B"] * WL["T"] / el, unit="tokens/s", cores=used, kind="oracle",
               sample=f"the whole workload ({WL['B']}x{WL['T']} tokens x {WL['H']} heads), fwd+bwd, fp64, "
                      f"threaded over heads ({used} threads used of {cores} cores)",
               seconds=el,
               single_thread=dict(value=WL["B"] * T1 / el1, unit="tokens/s", cores=1, seconds=el1,
                                  sample=f"first {T1} tokens x {WL['H']} heads, one thread"))
    if full:
        e1 = _oracle_time(inp, 1)
        out["single_thread_full"] = dict(value=WL["B"] * WL["T"] / e1, unit="tokens/s", cores=1, seconds=e1,
                                         sample="the whole workload, fwd+bwd, one thread")
        del inp, one
        wl3 = kin.WORKLOADS[3]
        f3 = kin.make_inputs(3, with_dO=False)
        ef = _oracle_time(f3, cores, bwd=False)
        ef1 = _oracle_time(f3, 1, bwd=False)
        out["fwd_long"] = dict(workload=wl3.name, threaded=dict(value=wl3.B * wl3.T / ef, unit="tokens/s",
                                                                 cores=min(cores, wl3.H), seconds=ef),
                               single_thread=dict(value=wl3.B * wl3.T / ef1, unit="tokens/s", cores=1,
                                                  seconds=ef1))
    return out


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    from delta_rule_linear_kron_b200 import inputs as kin
    from oracle import oracle
    cores = len(os.sched_getaffinity(0))
    inp = kin.make_inputs(4, T=REF_STEP_T, seed=1004)

    def step():
        oracle.fwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["c"], inp["logf"], inp["S0"], nthreads=cores)
        oracle.bwd(inp["q"], inp["k"], inp["v"], inp["beta"], inp["c"], inp["logf"], inp["S0"], inp["dO"],
                   nthreads=cores)

    for _ in range(args.warmup):
        step()
    t = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t
    value = WL["B"] * REF_STEP_T * args.steps / el
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": WORKLOAD_NAME, "B": WL["B"], "H": WL["H"], "T": REF_STEP_T, "dk": WL["dk"],
                       "dv": WL["dv"], "note": "each step: the first 512 tokens of the workload, all heads"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": min(cores, WL["H"]), "kind": "oracle",
                             "sample": f"{REF_STEP_T} tokens x {WL['H']} heads per step, fwd+bwd, fp64"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-fwd", action="store_true")
    ap.add_argument("--no-gated", action="store_true")
    ap.add_argument("--no-fused", action="store_true")
    ap.add_argument("--no-prologue", action="store_true")
    ap.add_argument("--no-gdn2", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-full", action="store_true",
                    help="also time the oracle on one thread over the whole workload, and on the long-context "
                         "forward workload (a few minutes)")
    args = ap.parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    import delta_rule_linear_kron_b200 as kd
    from delta_rule_linear_kron_b200 import inputs as kin

    ws_n, rank, local = dist_env()
    if ws_n > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks = load_peaks()
    B, H, T, dk, dv = WL["B"], WL["H"], WL["T"], WL["dk"], WL["dv"]

    def barrier():
        if ws_n > 1:
            dist.barrier()

    # ---- inputs (each rank its own batch) -------------------------------
    inp = kin.make_inputs(4, seed=rank_seed(1004, rank))
    bf, f32 = torch.bfloat16, torch.float32
    host = {n: torch.from_numpy(inp[n]).to(bf if n in ("q", "k", "v", "dO") else f32)
            for n in ("q", "k", "v", "dO", "beta", "c", "logf", "S0")}
    d = {n: t.to(dev) for n, t in host.items()}
    del inp
    fws = torch.empty(kd.workspace_size(kd.KD_WS_FWD_SAVE, B, H, T, dk, dv), dtype=torch.uint8, device=dev)
    bws = torch.empty(kd.workspace_size(kd.KD_WS_BWD, B, H, T, dk, dv), dtype=torch.uint8, device=dev)
    out = torch.empty((B, T, H, dv), dtype=bf, device=dev)

    def step(src):
        o, ST, _ = kd.fwd(src["q"], src["k"], src["v"], src["beta"], src["c"], src["logf"], src["S0"], out=out,
                          save=True, workspace=fws)
        g = kd.bwd(src["q"], src["k"], src["v"], src["beta"], src["c"], src["logf"], src["S0"], src["dO"],
                   fwd_workspace=fws, workspace=bws)
        return o, ST, g

    for _ in range(args.warmup):
        step(d)
    torch.cuda.synchronize()
    kd.device_status()
    barrier()
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.steps):
        step(d)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_total = max_over_ranks(e0.elapsed_time(e1), ws_n, dev)
    # per-kernel times: the same steps again with the library's CUDA-event
    # profiler (its events between launches are kept out of the headline timing)
    import ctypes
    kd.lib().kron_delta_profile_enable(1)
    kd.lib().kron_delta_profile_report(None, 0, 1)
    for _ in range(args.steps):
        step(d)
    torch.cuda.synchronize()
    buf = ctypes.create_string_buffer(1 << 16)
    kd.lib().kron_delta_profile_report(buf, len(buf), 1)
    kd.lib().kron_delta_profile_enable(0)
    per_kernel = {}
    for line in buf.value.decode().splitlines():
        name, n, ms = line.split()
        per_kernel[name] = dict(launches=int(n), ms=float(ms))
    launches = sum(v["launches"] for v in per_kernel.values())

    # ---- forward only: the long-context workload (B1 H16 T16384, nonzero S0)
    # and the B4 H16 T2048 workload (S0 = 0), each timed on its own ----------
    fwd_lines = {}
    if not args.no_fwd:
        for wl_i, key in ((3, "fwd_long"), (2, "fwd_B4")):
            wl = kin.WORKLOADS[wl_i]
            fi = kin.make_inputs(wl_i, seed=rank_seed(wl.seed, rank), with_dO=False)
            fd = {n: torch.from_numpy(fi[n]).to(dev, bf if n in ("q", "k", "v") else f32)
                  for n in ("q", "k", "v", "beta", "c", "logf")}
            fd["S0"] = None if fi["S0"] is None else torch.from_numpy(fi["S0"]).to(dev, f32)
            del fi
            fo = torch.empty((wl.B, wl.T, wl.H, wl.dv), dtype=bf, device=dev)
            fST = torch.empty((wl.B, wl.H, wl.dv, wl.dk), dtype=f32, device=dev)
            fw = torch.empty(kd.workspace_size(kd.KD_WS_FWD, wl.B, wl.H, wl.T, wl.dk, wl.dv), dtype=torch.uint8,
                             device=dev)

            def fcall():
                kd.fwd(fd["q"], fd["k"], fd["v"], fd["beta"], fd["c"], fd["logf"], fd["S0"], out=fo,
                       state_out=fST, save=False, workspace=fw)
            for _ in range(max(3, args.warmup)):
                fcall()
            torch.cuda.synchronize()
            barrier()
            f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            f0.record(stream)
            for _ in range(args.steps):
                fcall()
            f1.record(stream)
            torch.cuda.synchronize()
            barrier()
            fms = max_over_ranks(f0.elapsed_time(f1), ws_n, dev) / args.steps
            fu = wl.B * wl.H * wl.T
            fbytes = FWD_BYTES * fu + (2 if fd["S0"] is not None else 1) * wl.B * wl.H * wl.dk * wl.dv * 4
            fl = dict(workload=wl.name, ms=fms, tokens_per_s=job_throughput(ws_n, wl.B * wl.T, 1, fms),
                      hbm_frac=fbytes / (fms / 1e3) / 1e9 / peaks["hbm_gbs"],
                      tc_frac=FWD_FLOPS * fu / (fms / 1e3) / 1e12 / peaks["bf16_tflops"])
            fl["roofline_ms"] = 1e3 * max(fbytes / (peaks["hbm_gbs"] * 1e9),
                                          FWD_FLOPS * fu / (peaks["bf16_tflops"] * 1e12))
            fl["frac"] = fl["roofline_ms"] / fms
            fwd_lines[key] = fl
            del fd, fo, fST, fw
        kd.device_status()

    # ---- the same step with gated inputs: the forget gate as its bf16
    # pre-activation f_pre and a per-head exponent a_log, logf = e^a_log log
    # sigma(f_pre) formed inside the chunk kernels and df_pre, da_log in their
    # epilogues (fwd_gated(save) + bwd_gated), timed on its own ----------------
    gated = None
    if not args.no_gated:
        g_ = torch.Generator(device=dev)
        g_.manual_seed(rank_seed(3004, rank))
        f_pre = (torch.randn((B, T, H, dk), generator=g_, device=dev) + 3.0).to(bf)
        a_log = torch.rand((H,), generator=g_, device=dev) * 2 - 1
        gfw = torch.empty(kd.workspace_size(kd.KD_WS_FWD_GATED, B, H, T, dk, dv), dtype=torch.uint8, device=dev)
        gbw = torch.empty(kd.workspace_size(kd.KD_WS_BWD_GATED, B, H, T, dk, dv), dtype=torch.uint8, device=dev)

        def gated_step():
            kd.fwd_gated(d["q"], d["k"], d["v"], d["beta"], d["c"], f_pre, a_log, d["S0"], out=out, save=True,
                         workspace=gfw)
            kd.bwd_gated(d["q"], d["k"], d["v"], d["beta"], d["c"], f_pre, a_log, d["S0"], d["dO"],
                         fwd_workspace=gfw, workspace=gbw)
        for _ in range(max(3, args.warmup)):
            gated_step()
        torch.cuda.synchronize()
        barrier()
        q0, q1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        q0.record(stream)
        for _ in range(args.steps):
            gated_step()
        q1.record(stream)
        torch.cuda.synchronize()
        barrier()
        qms = max_over_ranks(q0.elapsed_time(q1), ws_n, dev) / args.steps
        kd.device_status()
        # inputs a step uploads: the plain step's with bf16 f_pre and a_log in place of fp32 logf
        h2d_plain = sum(t.numel() * t.element_size() for t in host.values())
        h2d_gated = (h2d_plain - host["logf"].numel() * host["logf"].element_size()
                     + f_pre.numel() * f_pre.element_size() + a_log.numel() * a_log.element_size())
        gated = dict(ms=qms, tokens_per_s=job_throughput(ws_n, B * T, 1, qms),
                     input_bytes_per_step=h2d_gated, plain_input_bytes_per_step=h2d_plain,
                     step="fwd_gated(save) + bwd_gated (bf16 f_pre, fp32 a_log [H]; outputs df_pre, da_log)")
        del f_pre, a_log, gfw, gbw

    # ---- the same step from raw projections and gate pre-activations: the
    # input prologue fused into the chunk kernels (fwd_fused(save) +
    # bwd_fused), against the unfused layer (prologue pass, fwd, bwd, prologue
    # backward pass), each timed on its own ---------------------------------
    fused = None
    if not args.no_fused:
        g_ = torch.Generator(device=dev)
        g_.manual_seed(rank_seed(5004, rank))
        rn = lambda *sh, m=0.0: torch.randn(sh, generator=g_, device=dev) + m  # noqa: E731
        raw = dict(q_raw=rn(B, T, H, dk).to(bf), k_raw=rn(B, T, H, dk).to(bf), v_raw=rn(B, T, H, dv).to(bf),
                   beta_pre=rn(B, T, H), c_pre=rn(B, T, H), f_pre=rn(B, T, H, dk, m=3.0).to(bf),
                   a_log=torch.rand((H,), generator=g_, device=dev) * 2 - 1)
        rorder = ("q_raw", "k_raw", "v_raw", "beta_pre", "c_pre", "f_pre", "a_log")
        ffw = torch.empty(kd.workspace_size(kd.KD_WS_FWD_FUSED, B, H, T, dk, dv), dtype=torch.uint8, device=dev)
        fbw = torch.empty(kd.workspace_size(kd.KD_WS_BWD_FUSED, B, H, T, dk, dv), dtype=torch.uint8, device=dev)
        pws = torch.empty(kd.workspace_size(kd.KD_WS_PROLOGUE_BWD, B, H, T, dk, dv), dtype=torch.uint8,
                          device=dev)

        def fused_step():
            kd.fwd_fused(*(raw[n] for n in rorder), 2.0, d["S0"], out=out, save=True, workspace=ffw)
            kd.bwd_fused(*(raw[n] for n in rorder), 2.0, d["S0"], d["dO"], fwd_workspace=ffw, workspace=fbw)

        def unfused_step():
            pp = kd.prologue_fwd(*(raw[n] for n in rorder), 2.0)
            pa = [pp[n] for n in ("q", "k", "v", "beta", "c", "logf")]
            kd.fwd(*pa, d["S0"], out=out, save=True, workspace=fws)
            gg = kd.bwd(*pa, d["S0"], d["dO"], fwd_workspace=fws, workspace=bws)
            kd.prologue_bwd(*(raw[n] for n in rorder), gg["dq"], gg["dk"], gg["dv"], gg["dbeta"], gg["dc"],
                            gg["dlogf"], 2.0, workspace=pws)
        fl = {}
        for key, fn in (("fused", fused_step), ("unfused", unfused_step)):
            for _ in range(max(3, args.warmup)):
                fn()
            torch.cuda.synchronize()
            barrier()
            q0, q1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            q0.record(stream)
            for _ in range(args.steps):
                fn()
            q1.record(stream)
            torch.cuda.synchronize()
            barrier()
            fl[key] = max_over_ranks(q0.elapsed_time(q1), ws_n, dev) / args.steps
        kd.device_status()
        fused = dict(ms=fl["fused"], tokens_per_s=job_throughput(ws_n, B * T, 1, fl["fused"]),
                     unfused_ms=fl["unfused"], unfused_tokens_per_s=job_throughput(ws_n, B * T, 1, fl["unfused"]),
                     step="fwd_fused(save) + bwd_fused from raw bf16 q, k, v, f_pre and fp32 beta_pre, c_pre, "
                          "a_log; unfused: prologue_fwd + fwd(save) + bwd + prologue_bwd")
        del raw, ffw, fbw, pws

    # ---- decode: 1000 consecutive in-place steps --------------------------
    decode = None
    if not args.no_decode:
        Bd, Hd = 256, 16
        dd = kin.decode_token_inputs_torch(args.decode_steps, B=Bd, H=Hd, seed=rank_seed(1005, rank), device=dev)
        S = dd["S"]
        o_dec = torch.empty((Bd, Hd, dv), dtype=bf, device=dev)
        for t in range(3):
            kd.decode(dd["q"][t], dd["k"][t], dd["v"][t], dd["beta"][t], dd["c"][t], dd["logf"][t], S, out=o_dec)
        torch.cuda.synchronize()
        barrier()
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        d0.record(stream)
        for t in range(args.decode_steps):
            kd.decode(dd["q"][t], dd["k"][t], dd["v"][t], dd["beta"][t], dd["c"][t], dd["logf"][t], S, out=o_dec)
        d1.record(stream)
        torch.cuda.synchronize()
        barrier()
        dms = max_over_ranks(d0.elapsed_time(d1), ws_n, dev)
        per_head = 2 * dv * dk * 4 + 2 * dk * 2 + dv * 2 + dk * 4 + 8 + dv * 2
        bytes_total = ws_n * args.decode_steps * Bd * Hd * per_head
        decode = dict(value=bytes_total / (dms / 1e3) / 1e9, unit="GB/s", steps=args.decode_steps,
                      us_per_step=1e3 * dms / args.decode_steps, B=Bd, H=Hd, d=dk,
                      bytes_per_head=per_head,
                      hbm_frac=(bytes_total / ws_n / (dms / 1e3) / 1e9) / peaks["hbm_gbs"])
        del dd, S
    # ---- input prologue (raw projections -> q, k, v, beta, c, logf) and its
    # backward, on this workload's shape, timed on their own --------------
    prologue = None
    if not args.no_prologue:
        g_ = torch.Generator(device=dev)
        g_.manual_seed(rank_seed(2004, rank))
        rn = lambda *sh, m=0.0: torch.randn(sh, generator=g_, device=dev) + m  # noqa: E731
        pr = dict(q_raw=rn(B, T, H, dk).to(bf), k_raw=rn(B, T, H, dk).to(bf), v_raw=rn(B, T, H, dv).to(bf),
                  beta_pre=rn(B, T, H), c_pre=rn(B, T, H), f_pre=rn(B, T, H, dk, m=3.0).to(bf),
                  a_log=torch.rand((H,), generator=g_, device=dev) * 2 - 1)
        up = dict(dq=rn(B, T, H, dk).to(bf), dk=rn(B, T, H, dk).to(bf), dv=rn(B, T, H, dv).to(bf),
                  dbeta=rn(B, T, H), dc=rn(B, T, H), dlogf=rn(B, T, H, dk))
        ep = dict(o=(0.1 * rn(B, T, H, dv)).to(bf), g=rn(B, T, H, dv).to(bf), w=1 + 0.1 * rn(dv),
                  dy=rn(B, T, H, dv).to(bf))
        ews = torch.empty(kd.workspace_size(kd.KD_WS_EPILOGUE_BWD, B, H, T, dk, dv), dtype=torch.uint8,
                          device=dev)
        y_ep = torch.empty_like(ep["o"])
        pws = torch.empty(kd.workspace_size(kd.KD_WS_PROLOGUE_BWD, B, H, T, dk, dv), dtype=torch.uint8,
                          device=dev)
        order = ("q_raw", "k_raw", "v_raw", "beta_pre", "c_pre", "f_pre", "a_log")
        times = {}
        for name in ("prologue_fwd", "prologue_bwd", "epilogue_fwd", "epilogue_bwd"):
            def call():
                if name == "prologue_fwd":
                    kd.prologue_fwd(*(pr[n] for n in order), 2.0)
                elif name == "prologue_bwd":
                    kd.prologue_bwd(*(pr[n] for n in order), up["dq"], up["dk"], up["dv"], up["dbeta"], up["dc"],
                                    up["dlogf"], 2.0, workspace=pws)
                elif name == "epilogue_fwd":
                    kd.epilogue_fwd(ep["o"], ep["g"], ep["w"], out=y_ep)
                else:
                    kd.epilogue_bwd(ep["o"], ep["g"], ep["w"], ep["dy"], workspace=ews)
            for _ in range(3):
                call()
            torch.cuda.synchronize()
            barrier()
            p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            p0.record(stream)
            for _ in range(args.steps):
                call()
            p1.record(stream)
            torch.cuda.synchronize()
            barrier()
            ms = max_over_ranks(p0.elapsed_time(p1), ws_n, dev) / args.steps
            pb = pass_bytes(name)
            gbs = pb * B * H * T / (ms / 1e3) / 1e9
            times[name] = dict(ms=ms, algorithmic_bytes_per_launch=pb * B * H * T, achieved_gbs=gbs,
                               hbm_frac=gbs / peaks["hbm_gbs"])
        kd.device_status()
        prologue = dict(times, note="timed alone, not part of the step; each bwd time includes its small "
                                    "fixed-order reduction launch (da_log, dw)")
        del pr, up, ep
    # ---- Gated DeltaNet-2 rule on the same shape: fwd + bwd, timed on its own
    gdn2 = None
    if not args.no_gdn2:
        g_ = torch.Generator(device=dev)
        g_.manual_seed(rank_seed(4004, rank))

        def unit_(*sh):
            x = torch.randn(sh, generator=g_, device=dev)
            return (x / x.norm(dim=-1, keepdim=True)).to(bf)
        gi = dict(q=unit_(B, T, H, dk), k=unit_(B, T, H, dk), v=unit_(B, T, H, dv),
                  b=torch.sigmoid(torch.randn((B, T, H, dk), generator=g_, device=dev)),
                  w=torch.sigmoid(torch.randn((B, T, H, dv), generator=g_, device=dev)),
                  loga=-torch.nn.functional.softplus(torch.randn((B, T, H, dk), generator=g_, device=dev) - 4.0))
        gdO = torch.randn((B, T, H, dv), generator=g_, device=dev).to(bf)
        gS0 = torch.randn((B, H, dv, dk), generator=g_, device=dev)
        gS0 = gS0 / gS0.norm(dim=(-2, -1), keepdim=True)
        gfws = torch.empty(kd.workspace_size(kd.KD_WS_GDN2_FWD, B, H, T, dk, dv), dtype=torch.uint8, device=dev)
        gbws = torch.empty(kd.workspace_size(kd.KD_WS_GDN2_BWD, B, H, T, dk, dv), dtype=torch.uint8, device=dev)
        gorder = ("q", "k", "v", "b", "w", "loga")

        def gstep():
            kd.gdn2_fwd(*(gi[n] for n in gorder), gS0, workspace=gfws)
            kd.gdn2_bwd(*(gi[n] for n in gorder), gS0, gdO, fwd_workspace=gfws, workspace=gbws)
        gsteps = max(1, min(args.steps, 5))
        for _ in range(3):
            gstep()
        torch.cuda.synchronize()
        barrier()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(gsteps):
            gstep()
        g1.record(stream)
        torch.cuda.synchronize()
        barrier()
        gms = max_over_ranks(g0.elapsed_time(g1), ws_n, dev) / gsteps
        kd.lib().kron_delta_profile_enable(1)
        kd.lib().kron_delta_profile_report(None, 0, 1)
        gstep()
        torch.cuda.synchronize()
        gbuf = ctypes.create_string_buffer(1 << 14)
        kd.lib().kron_delta_profile_report(gbuf, len(gbuf), 1)
        kd.lib().kron_delta_profile_enable(0)
        gk = {ln.split()[0]: float(ln.split()[2]) for ln in gbuf.value.decode().splitlines()}
        kd.device_status()
        del gi, gdO, gfws, gbws
        # decode: 100 consecutive in-place steps, B=256, H=16, d=128 (the decode workload's shape)
        Bd, Hd, nd = 256, 16, 100

        def unit3(*sh):
            x = torch.randn(sh, generator=g_, device=dev)
            return (x / x.norm(dim=-1, keepdim=True)).to(bf)
        dq_, dk_, dvv = unit3(nd, Bd, Hd, dk), unit3(nd, Bd, Hd, dk), unit3(nd, Bd, Hd, dv)
        db_ = torch.sigmoid(torch.randn((nd, Bd, Hd, dk), generator=g_, device=dev))
        dw_ = torch.sigmoid(torch.randn((nd, Bd, Hd, dv), generator=g_, device=dev))
        dla = -torch.nn.functional.softplus(torch.randn((nd, Bd, Hd, dk), generator=g_, device=dev) - 4.0)
        Sd = torch.randn((Bd, Hd, dv, dk), generator=g_, device=dev) * (1.0 / 128.0) ** 0.5
        od = torch.empty((Bd, Hd, dv), dtype=bf, device=dev)
        for t in range(3):
            kd.gdn2_decode(dq_[t], dk_[t], dvv[t], db_[t], dw_[t], dla[t], Sd, out=od)
        torch.cuda.synchronize()
        barrier()
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        d0.record(stream)
        for t in range(nd):
            kd.gdn2_decode(dq_[t], dk_[t], dvv[t], db_[t], dw_[t], dla[t], Sd, out=od)
        d1.record(stream)
        torch.cuda.synchronize()
        barrier()
        dms = max_over_ranks(d0.elapsed_time(d1), ws_n, dev)
        per_head = 2 * dv * dk * 4 + 2 * dk * 2 + dv * 2 + 2 * dk * 4 + dv * 4 + dv * 2
        gdec = dict(value=ws_n * nd * Bd * Hd * per_head / (dms / 1e3) / 1e9, unit="GB/s", steps=nd,
                    us_per_step=1e3 * dms / nd, B=Bd, H=Hd, bytes_per_head=per_head,
                    hbm_frac=(nd * Bd * Hd * per_head / (dms / 1e3) / 1e9) / peaks["hbm_gbs"])
        del dq_, dk_, dvv, db_, dw_, dla, Sd
        alu_peak = fp32_alu_peak_tflops(1965.0)
        gkr = {}
        for name, kms in gk.items():
            f = gdn2_kernel_flops(name)
            if f is None or kms <= 0:
                continue
            ach = f * B * H * T / (kms / 1e3) / 1e12
            tcn = name.endswith("_tc")
            pk = peaks["bf16_tflops"] if tcn else alu_peak
            gkr[name] = dict(bound="tensor" if tcn else "alu", achieved=ach, peak=pk, unit="TFLOP/s",
                             frac=ach / pk, algorithmic_flops_per_launch=f * B * H * T, ms=kms)
        top = max(gkr, key=lambda n: gkr[n]["ms"]) if gkr else None
        gdn2 = dict(value=job_throughput(ws_n, B * T, 1, gms), unit="tokens/s", ms_per_step=gms,
                    step="gdn2_fwd + gdn2_bwd (bf16 q/k/v/dO, fp32 gates; chunk products on tcgen05)",
                    per_kernel_ms=gk, kernel_rooflines=gkr,
                    roofline=None if top is None else dict(
                        kernel=top, **gkr[top],
                        peak_note=("measured bf16 dense (burst)" if gkr[top]["bound"] == "tensor"
                                   else "148 SMs x 128 FP32 lanes x 2 x 1965 MHz")),
                    decode=gdec)
    clocks = sampler.stop()

    # ---- end to end through the public API with pinned host buffers -----
    def end_to_end(host_in, step_fn):
        # Every step copies its inputs from pinned host memory and reads its
        # results back inside the timed region.  Step s+1's inputs travel on a
        # copy stream into the other of two device buffers while step s
        # computes; a buffer is refilled only after the step that read it ended.
        pinned = {n: t.pin_memory() for n, t in host_in.items()}
        staged = [{n: torch.empty_like(t, device=dev) for n, t in host_in.items()} for _ in range(2)]
        out_h = torch.empty((B, T, H, dv), dtype=bf).pin_memory()
        dS0_h = torch.empty((B, H, dv, dk), dtype=f32).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in pinned.values())
        d2h = out_h.numel() * out_h.element_size() + dS0_h.numel() * dS0_h.element_size()
        copy = torch.cuda.Stream(device=dev)
        loaded = [torch.cuda.Event(), torch.cuda.Event()]
        consumed = [torch.cuda.Event(), torch.cuda.Event()]
        barrier()
        torch.cuda.synchronize()
        x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        x0.record(stream)
        copy.wait_stream(stream)

        def upload(slot, after_step):
            with torch.cuda.stream(copy):
                if after_step:
                    copy.wait_event(consumed[slot])
                for n, t in staged[slot].items():
                    t.copy_(pinned[n], non_blocking=True)
                loaded[slot].record(copy)
        upload(0, False)
        for si in range(args.e2e_steps):
            slot = si % 2
            if si + 1 < args.e2e_steps:
                upload(1 - slot, si >= 1)
            stream.wait_event(loaded[slot])
            o, dS0 = step_fn(staged[slot])
            consumed[slot].record(stream)
            out_h.copy_(o, non_blocking=True)
            dS0_h.copy_(dS0, non_blocking=True)
        x1.record(stream)
        torch.cuda.synchronize()
        barrier()
        xms = max_over_ranks(x0.elapsed_time(x1), ws_n, dev)
        del staged
        return dict(value=job_throughput(ws_n, B * T, args.e2e_steps, xms), unit="tokens/s",
                    h2d_bytes_per_step=h2d, d2h_bytes_per_step=d2h, ms_per_step=xms / args.e2e_steps,
                    h2d_gbs=h2d * args.e2e_steps / (xms / 1e3) / 1e9,
                    pipelining="next step's H2D on a copy stream overlaps this step's compute; D2H after it")

    e2e = e2e_gated = None
    if not args.no_e2e:
        def plain_e2e_step(src):
            o, _, g = step(src)
            return o, g["dS0"]
        e2e = end_to_end(host, plain_e2e_step)
        # the same step through the gated entry points: the forget gate
        # uploaded as its bf16 pre-activation (and a_log per head) in place of
        # the fp32 log-decay
        gen = torch.Generator()
        gen.manual_seed(rank_seed(5004, rank))
        ghost = {n: t for n, t in host.items() if n != "logf"}
        ghost["f_pre"] = (torch.randn((B, T, H, dk), generator=gen) + 3.0).to(bf)
        ghost["a_log"] = torch.rand((H,), generator=gen) * 2 - 1
        e_fw = torch.empty(kd.workspace_size(kd.KD_WS_FWD_GATED, B, H, T, dk, dv), dtype=torch.uint8, device=dev)
        e_bw = torch.empty(kd.workspace_size(kd.KD_WS_BWD_GATED, B, H, T, dk, dv), dtype=torch.uint8, device=dev)

        def gated_e2e_step(src):
            o, _, _ = kd.fwd_gated(src["q"], src["k"], src["v"], src["beta"], src["c"], src["f_pre"], src["a_log"],
                                   src["S0"], out=out, save=True, workspace=e_fw)
            g = kd.bwd_gated(src["q"], src["k"], src["v"], src["beta"], src["c"], src["f_pre"], src["a_log"],
                             src["S0"], src["dO"], fwd_workspace=e_fw, workspace=e_bw)
            return o, g["dS0"]
        for _ in range(2):
            gated_e2e_step({n: t.to(dev) for n, t in ghost.items()})
        torch.cuda.synchronize()
        e2e_gated = end_to_end(ghost, gated_e2e_step)
        e2e_gated["step"] = "fwd_gated(save) + bwd_gated: bf16 f_pre and a_log [H] uploaded in place of fp32 logf"
        del e_fw, e_bw, ghost
        kd.device_status()

    value = job_throughput(ws_n, B * T, args.steps, ms_total)

    # ---- rooflines against the method's algorithmic work -----------------
    # Per kernel: the method rows it executes (flops against the measured
    # burst bf16 GEMM peak: the timed region is tens of ms) and the method
    # bytes it must move (against the measured HBM copy bandwidth); the
    # binding bound is the larger of the two times.  For the step: 524,288
    # flops and 4,376 B per token-head against ms_per_step.
    units = B * H * T  # token-heads per launch of every per-step kernel
    tc_peak, hbm_peak = peaks["bf16_tflops"], peaks["hbm_gbs"]
    kernels = {}
    for name, v in per_kernel.items():
        w = method_work(name)
        if w is None or v["launches"] == 0:
            continue
        avg_s = v["ms"] / v["launches"] / 1e3
        t_c = w["flops"] * units / (tc_peak * 1e12)
        t_m = w["bytes"] * units / (hbm_peak * 1e9)
        io = kernel_io_bytes(name) * units
        tr = ncu_traffic(name)
        k = dict(rows=w["rows"], avg_launch_ms=avg_s * 1e3, algorithmic_flops_per_launch=w["flops"] * units,
                 algorithmic_bytes_per_launch=w["bytes"] * units, design_io_bytes_per_launch=io, traffic=tr,
                 traffic_ratio=None if tr is None else tr / (w["bytes"] * units))
        if t_c >= t_m:
            ach = w["flops"] * units / avg_s / 1e12
            k.update(bound="tensor", achieved=ach, peak=tc_peak, unit="TFLOP/s", frac=ach / tc_peak)
        else:
            ach = w["bytes"] * units / avg_s / 1e9
            k.update(bound="hbm", achieved=ach, peak=hbm_peak, unit="GB/s", frac=ach / hbm_peak)
        kernels[name] = k
    roofline = None
    if kernels:
        top = max(kernels, key=lambda n: per_kernel[n]["ms"])
        k = kernels[top]
        roofline = dict(kernel=top, rows=k["rows"], bound=k["bound"], achieved=k["achieved"], peak=k["peak"],
                        unit=k["unit"], frac=k["frac"], traffic=k["traffic"], avg_launch_ms=k["avg_launch_ms"],
                        algorithmic_flops_per_launch=k["algorithmic_flops_per_launch"],
                        algorithmic_bytes_per_launch=k["algorithmic_bytes_per_launch"],
                        peak_note=("measured HBM copy bandwidth" if k["bound"] == "hbm" else
                                   "measured burst bf16 GEMM") + " (" + peaks["source"] + ")",
                        sm_mhz_median=clocks["sm_mhz"])
    step_s = ms_total / args.steps / 1e3
    st_bytes = STEP_BYTES * units + 3 * B * H * dk * dv * 4
    st_flops = STEP_FLOPS * units
    traffic_all = [kernels[n]["traffic"] for n in kernels]
    roofline_step = dict(
        flops_per_token_head=STEP_FLOPS, bytes_per_token_head=STEP_BYTES, ms=step_s * 1e3,
        achieved_gbs=st_bytes / step_s / 1e9, hbm_frac=st_bytes / step_s / 1e9 / hbm_peak,
        achieved_tflops=st_flops / step_s / 1e12, tc_frac=st_flops / step_s / 1e12 / tc_peak,
        roofline_ms=1e3 * max(st_bytes / (hbm_peak * 1e9), st_flops / (tc_peak * 1e12)),
        bound="hbm" if st_bytes / hbm_peak / 1e9 >= st_flops / tc_peak / 1e12 else "tensor",
        traffic_bytes=(sum(traffic_all) if traffic_all and None not in traffic_all else None))
    roofline_step["frac"] = roofline_step["roofline_ms"] / (step_s * 1e3)
    roofline_step["traffic_ratio"] = (None if roofline_step["traffic_bytes"] is None
                                      else roofline_step["traffic_bytes"] / st_bytes)

    cpu = None
    if rank == 0 and ws_n == 1 and not args.no_cpu_baseline:
        cpu = oracle_baseline(full=args.cpu_full)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws_n, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_total / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": WORKLOAD_NAME, "B": B, "H": H, "T": T, "dk": dk, "dv": dv, "chunk": CHUNK,
                           "global_batch": B * ws_n, "seq_len": T, "parallelism": f"dp{ws_n}",
                           "step": "fwd(save) + bwd", "l2": "inputs larger than L2 (no flush)"},
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "e2e_gated": e2e_gated,
                "gpu_launches": launches,
                "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                           "reasons": clocks["reasons"], "samples": clocks["samples"]},
                "peaks": peaks,
                "per_kernel_ms": {k: v["ms"] / max(1, args.steps) for k, v in per_kernel.items()},
                "kernel_rooflines": kernels,
                "prologue_epilogue": prologue,
                "gdn2": gdn2,
                # compact summaries last (a truncated tail of the line keeps them)
                "roofline_step": roofline_step,
                "fwd_long": fwd_lines.get("fwd_long"), "fwd_B4": fwd_lines.get("fwd_B4"),
                "gated_step": gated,
                "fused_step": fused,
                "gdn2_step": None if gdn2 is None else dict(ms=gdn2["ms_per_step"], tokens_per_s=gdn2["value"],
                                                            decode_gbs=gdn2["decode"]["value"],
                                                            decode_hbm_frac=gdn2["decode"]["hbm_frac"]),
                "decode": decode}
        print(json.dumps(line), flush=True)
    if ws_n > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
