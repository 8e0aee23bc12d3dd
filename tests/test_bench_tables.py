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
    assert bench.kernel_work("prologue_fwd")["bytes"] == 4 * act + 8 + 3 * act + lf + 8 == 2320
    assert bench.kernel_work("prologue_bwd")["bytes"] == 3352
    assert bench.kernel_work("epilogue_fwd")["bytes"] == 3 * act == 768
    assert bench.kernel_work("epilogue_bwd")["bytes"] == 5 * act == 1280


def test_fp32_alu_peak():
    assert abs(bench.fp32_alu_peak_tflops(1965.0) - 148 * 128 * 2 * 1.965e9 / 1e12) < 1e-9
