"""The benchmark's algorithmic-work tables, checked against the closed forms
they are derived from (CPU only)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_gdn2_flops_match_the_chunk_products():
    d, C = 128, 64
    f = {n: bench.gdn2_kernel_flops(n, d, C) for n in
         ("gdn2_prep", "gdn2_chain", "gdn2_out", "gdn2_bchain", "gdn2_bpost_a", "gdn2_bpost_b")}
    # forward: T, P, W, U' (4 C x d products), U and the state update (2 d x d), O (one of each)
    assert f["gdn2_prep"] + f["gdn2_chain"] + f["gdn2_out"] == 5 * 2 * C * d + 3 * 2 * d * d
    # backward: 6 d x d products (P^T dO is C x d) and 10 C x d products
    back = f["gdn2_bchain"] + f["gdn2_bpost_a"] + f["gdn2_bpost_b"]
    assert back == 6 * 2 * d * d + 10 * 2 * C * d
    assert bench.gdn2_kernel_flops("gdn2_decode_kernel") is None


def test_prologue_epilogue_bytes_per_token_head():
    act, lf = 256, 512  # bf16 row of 128, fp32 row of 128
    assert bench.pass_bytes("prologue_fwd") == 4 * act + 8 + 3 * act + lf + 8 == 2320
    assert bench.pass_bytes("prologue_bwd") == 3352
    assert bench.pass_bytes("epilogue_fwd") == 3 * act == 768
    assert bench.pass_bytes("epilogue_bwd") == 5 * act == 1280


def test_step_kernels_carry_the_method_flops_once():
    """Forward kernels execute rows a1-a8 (163,840 flops per token-head), the
    backward's a9-a10 (360,448): each row's contractions counted once."""
    d, C = 128, 64
    fwd = ("fwd_prep_tc", "fwd_cross_tc", "fwd_chain_tc", "fwd_out_tc")
    bwd = ("bwd_pre_tc", "bwd_chain_tc", "bwd_post_tc")
    f = sum(bench.method_work(n)["flops"] for n in fwd)
    b = sum(bench.method_work(n)["flops"] for n in bwd)
    assert f == 6 * d * d + 4 * C * (2 * d) == bench.FWD_FLOPS == 163840
    assert b == 14 * d * d + 8 * C * (2 * d) == 360448
    assert f + b == bench.STEP_FLOPS
    # the chains: a5 + a7 forward, a9 (three d x d x C contractions) backward
    assert bench.method_work("fwd_chain_tc")["flops"] == 2 * 2 * d * d
    assert bench.method_work("bwd_chain_tc")["flops"] == 3 * 2 * d * d
    # no kernel is credited with more method bytes than its pass of the operation moves
    assert all(bench.method_work(n)["bytes"] <= bench.FWD_BYTES for n in fwd)
    assert all(bench.method_work(n)["bytes"] <= bench.STEP_BYTES - bench.FWD_BYTES for n in bwd)
    assert bench.STEP_BYTES == 3 * 256 + 8 + 512 + 256 + (3 * 256 + 8 + 512 + 256) + 3 * 256 + 8 + 512


def test_fp32_alu_peak():
    assert abs(bench.fp32_alu_peak_tflops(1965.0) - 148 * 128 * 2 * 1.965e9 / 1e12) < 1e-9
