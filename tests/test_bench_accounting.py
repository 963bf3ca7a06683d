"""bench.py's accounting of the work it reports: launches per forward (its
gpu_launches claim) and the algorithmic FLOPs and bytes behind its roofline
fractions, worked out by hand for the decode and prefill layers."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from mixture_experts_layer_28_b200 import workloads as wl  # noqa: E402


def test_launches_per_forward():
    # router GEMM, route, assign, permute, gate/up, down, combine
    assert bench.kernels_per_forward(wl.get("prefill")) == 7
    # at most 64 tokens: the two expert GEMMs are one kernel
    assert bench.kernels_per_forward(wl.get("decode")) == 6
    assert bench.kernels_per_forward(wl.get("tiny", T=64)) == 6
    assert bench.kernels_per_forward(wl.get("tiny", T=65)) == 7
    # no FFN experts: no dispatch to experts, no GEMM (assign still clears slots)
    assert bench.kernels_per_forward(wl.get("tiny", N=0, Z=12, K=3)) == 4


def test_routing_stats_counts_ffn_pairs_and_hit_experts():
    w = wl.get("tiny")                      # N = 8 FFN experts, Z = 4
    cnt = np.array([5, 0, 3, 0, 0, 0, 0, 9, 100, 100, 100, 100])
    st = bench.routing_stats(w, cnt)
    assert st["ffn_pairs"] == 17 and st["experts_hit"] == 3 and st["max_load"] == 9
    assert abs(st["zero_pick_fraction"] - (1 - 17 / (w.T * w.K))) < 1e-12


def test_decode_roofline_bytes():
    """Decode layer: 30 of 512 experts hit by 460 (token, expert) pairs; the
    one expert-GEMM kernel must stream the three 6144 x 2048 bf16 matrices of
    each hit expert once, plus the permuted tokens, H written and read back,
    and Y: 2.279 GB (the figure its ncu DRAM traffic is compared with)."""
    w = wl.get("decode")
    rf = bench.roofline_numbers(w, dict(ffn_pairs=460, experts_hit=30), None)
    weights = 30 * 3 * 6144 * 2048 * 2
    acts = 460 * 6144 * 2 + 2 * 460 * 2048 * 2 + 460 * 6144 * 2
    assert rf["B_gateup"] + rf["B_down"] == weights + acts
    assert abs((weights + acts) / 1e9 - 2.279) < 0.001
    # SwiGLU: 2 d I multiply-adds for gate and up, d I for down, per pair
    assert rf["F_gateup"] == 4.0 * 6144 * 2048 * 460
    assert rf["F_down"] == 2.0 * 6144 * 2048 * 460
    # the layer touches each hit expert's weights, the router (W_r and the
    # bias) and x in and out once
    assert rf["B_layer"] == weights + 768 * 6144 * 2 + 768 * 4 + 2 * 64 * 6144 * 2


def test_prefill_executed_ffn_flops():
    """Prefill layer, 137,695 FFN pairs: 6 d I FLOPs per pair, 1.04e13 in all
    (69% of the measured 1662 TFLOP/s bf16 burst peak at 9.06 ms)."""
    w = wl.get("prefill")
    rf = bench.roofline_numbers(w, dict(ffn_pairs=137695, experts_hit=57), None)
    assert rf["F_layer"] == 6.0 * 6144 * 2048 * 137695
    assert abs(rf["F_layer"] / 9.06e-3 / 1e12 / 1662.4 - 0.69) < 0.005
