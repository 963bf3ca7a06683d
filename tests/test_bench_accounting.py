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
    # at most 64 tokens: the router GEMM, then one grid that routes,
    # dispatches, runs both expert GEMMs and combines
    assert bench.kernels_per_forward(wl.get("decode")) == 2
    assert bench.kernels_per_forward(wl.get("tiny", T=64)) == 2
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


def _pk():
    return dict(hbm=6457.4, bf16=1662.4, bf16_sus=1374.8, src="measured")


def test_short_regions_use_the_burst_peak():
    """A timed region of 20 prefill steps (~0.2 s) holds kernels to the burst
    bf16 peak; only regions of seconds use the sustained one."""
    assert bench.bf16_peak(_pk(), 0.18)[0] == 1662.4
    assert bench.bf16_peak(_pk(), 5.0)[0] == 1374.8


def test_prefill_gateup_roofline_against_burst_peak():
    """The gate/up GEMM of the prefill layer: 4 d I FLOPs per pair over
    137,695 pairs in 5.2495 ms is 1320 TFLOP/s, 0.794 of the 1662.4 burst
    peak (0.960 of the sustained one)."""
    w = wl.get("prefill")
    rf = bench.roofline_numbers(w, dict(ffn_pairs=137695, experts_hit=57), None)
    plan = dict(expert_gemms_one_grid=0)
    per = {"router_gemm": 0.15, "gateup_gemm": 5.2495, "down_gemm": 2.83}
    roof = bench.kernel_roofline(w, rf, plan, per, _pk(), region_s=0.18)
    assert roof["bound"] == "tensor" and roof["kernel"] == "gateup_gemm"
    assert abs(roof["achieved"] - 1320.2) < 0.5
    assert abs(roof["frac"] - 0.794) < 0.001
    assert abs(roof["frac_of_sustained_peak"] - 0.960) < 0.001


def test_decode_one_grid_roofline_is_hbm_bound():
    """Decode: the one kernel running both expert GEMMs moves 2.279 GB; at
    0.35 ms that is 6.51 TB/s, against the 6457.4 GB/s measured copy peak and
    the 7.7 TB/s nominal figure."""
    w = wl.get("decode")
    rf = bench.roofline_numbers(w, dict(ffn_pairs=460, experts_hit=30), None)
    roof = bench.kernel_roofline(w, rf, dict(expert_gemms_one_grid=1),
                                 {"gateup_gemm": 0.35, "route": 0.02}, _pk(), region_s=1.0)
    assert roof["bound"] == "hbm" and roof["kernel"].startswith("gateup_down_gemm")
    assert abs(roof["achieved"] - 2.279e9 / 0.35e-3 / 1e9) < 5
    assert abs(roof["frac_of_nominal_hbm"] - roof["achieved"] / 7700.0) < 1e-12


def test_decode_step_kernel_counts_its_phases_bytes():
    """Decode with the whole step in the one grid: besides the expert GEMMs'
    2.279 GB the kernel reads the router's 24 K slices of partial logits
    (24 x 64 x 768 fp32), writes picks, gates and slots (64 x 12 x 3 x 4 B)
    and zsum, reads x twice, writes the 460 permuted rows, reads the 460 Y
    rows back and writes out: 18.4 MB more."""
    w = wl.get("decode")
    rf = bench.roofline_numbers(w, dict(ffn_pairs=460, experts_hit=30), None, splits=24)
    phases = (24 * 64 * 768 * 4 + 64 * 12 * 12 + 64 * 4 + 2 * 64 * 6144 * 2 + 460 * 6144 * 2
              + 460 * 6144 * 2 + 64 * 6144 * 2)
    assert rf["B_phases"] == phases
    assert abs(phases / 1e6 - 18.4) < 0.05
    plan = dict(expert_gemms_one_grid=1, one_grid_step=1)
    roof = bench.kernel_roofline(w, rf, plan, {"gateup_gemm": 0.36}, _pk(), region_s=1.0)
    assert roof["kernel"].startswith("decode_step")
    assert roof["algorithmic_bytes"] == rf["B_gateup"] + rf["B_down"] + phases
    assert abs(roof["achieved"] - roof["algorithmic_bytes"] / 0.36e-3 / 1e9) < 1e-6


def test_clock_samples_outside_the_region_are_dropped():
    c = bench.ClockSampler(0)
    c.lines = [
        "2026/12/02 10:00:00.000, 0, 600, 1965, 200, 0x0, Not Active, Not Active, Not Active, Not Active",
        "2026/12/02 10:00:01.000, 0, 1965, 1965, 900, 0x4, Not Active, Not Active, Not Active, Active",
        "2026/12/02 10:00:01.100, 0, 1900, 1965, 950, 0x4, Not Active, Not Active, Not Active, Active",
        "2026/12/02 10:00:03.000, 0, 700, 1965, 250, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    t0 = bench.ClockSampler._stamp("2026/12/02 10:00:00.900")
    t1 = bench.ClockSampler._stamp("2026/12/02 10:00:01.200")
    s = c.summary(t0, t1)
    assert s["samples"] == 2 and s["sm_mhz"] == (1965 + 1900) / 2
    assert s["reasons"] == ["sw_power_cap"] and s["samples_outside_region"] == 2


def test_fp8_layer_bytes_and_peak():
    """FP8 gate/up: weights and tokens at one byte plus a scale byte per 32
    elements; the down projection stays bf16.  The decode layer with 30 hit
    experts then touches 30 x (2 x 2048 x 6144 x 33/32 + 6144 x 2048 x 2)
    bytes of expert weights; its gate/up kernel is held to twice the bf16
    peak."""
    w = wl.get("decode")
    rf = bench.roofline_numbers(w, dict(ffn_pairs=460, experts_hit=30), None, fp8=True)
    weights = 30 * (2 * 2048 * 6144 * 33 / 32 + 6144 * 2048 * 2)
    assert rf["B_layer"] == weights + 768 * 6144 * 2 + 768 * 4 + 2 * 64 * 6144 * 2
    assert rf["B_gateup"] == 30 * 2 * 2048 * 6144 * 33 / 32 + 460 * 6144 * 33 / 32 + 460 * 2048 * 2
    assert bench.tensor_peak(_pk(), 0.5, fp8=True)[0] == 2 * 1662.4
    # the layer's tensor bound counts gate/up FLOPs at the FP8 rate
    lr = bench.layer_roofline(rf, _pk(), 1.0, 0.5)
    t_f = (rf["F_gateup"] / 2 + rf["F_down"]) / 1662.4e12
    t_b = rf["B_layer"] / 6457.4e9
    assert abs(lr["roofline_ms"] - max(t_f, t_b) * 1e3) < 1e-12
