"""Host logic of the multi-GPU path, run as two CPU processes over gloo.

The mixer shards over (batch, head) units with no data-path collective: each
rank runs its own batch of the workload's shape (weak scaling), and the only
cross-rank steps are the barrier and the max-over-ranks reduction of the
timed region, from which the whole-job throughput is formed.  These tests run
exactly those functions of bench.py with world size 2 on the gloo backend.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime

    import torch
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    ws_n, r, local = bench.dist_env()
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    dev = torch.device("cpu")
    # each rank times a different amount of work; the job takes the slowest rank's time
    my_ms = 10.0 + 5.0 * r
    ms_total = bench.max_over_ranks(my_ms, ws_n, dev)
    dist.barrier()
    value = bench.job_throughput(ws_n, 16384, 4, ms_total)
    seeds = bench.rank_seed(1004, r)
    with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
        json.dump(dict(ws=ws_n, rank=r, local=local, ms=ms_total, value=value, seed=seeds), f)
    dist.destroy_process_group()


def test_two_ranks_gloo_max_over_ranks_and_throughput(tmp_path):
    import torch.multiprocessing as mp
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    for r, x in enumerate(res):
        assert x["ws"] == 2 and x["rank"] == r and x["local"] == r
        assert x["ms"] == 15.0  # the slowest rank's time on every rank
        # 2 ranks x 16384 tokens x 4 steps in 15 ms
        assert abs(x["value"] - 2 * 16384 * 4 / 0.015) < 1e-6 * x["value"]
    assert res[0]["seed"] != res[1]["seed"]  # each rank draws its own batch


def test_rank_inputs_are_distinct_batches():
    import bench
    from delta_rule_linear_kron_b200 import inputs as kin
    a = kin.make_inputs(1, T=64, seed=bench.rank_seed(1001, 0))
    b = kin.make_inputs(1, T=64, seed=bench.rank_seed(1001, 1))
    assert a["q"].shape == b["q"].shape
    assert (a["q"] != b["q"]).any()


def test_reference_arm_runs_on_rank_zero_only():
    """Under torchrun the oracle arm prints from rank 0; other ranks exit 0 without work."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_single_rank_reduction_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1, None) == 3.5
    assert bench.job_throughput(1, 100, 2, 1000.0) == 200.0
