#!/usr/bin/env python
"""Benchmark of the B200 MoE layer with zero-computation experts.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference]

One step is one forward of the whole layer (router GEMM, routing, dispatch,
gate/up and down expert GEMMs, combine) over one batch of T synthetic tokens,
through the C ABI (moe_zc_forward).  The default workload is the
LongCat-Flash-shaped prefill layer (T=16384, d=6144, N=512 SwiGLU experts with
I=2048, Z=256 zero experts, K=12, ~30% zero-expert picks); --workload picks
another (tiny, small, decode, skewed20/40/60).

Timing: W untimed warm-up steps, then K steps between CUDA events on the
launching stream, with a barrier and a device synchronize on both sides; the
max over ranks is taken.  The expert weights the batch touches (several GB at
prefill) are far larger than the 126 MB L2, so no L2 flush is done between
steps.  With N > 1 GPUs each rank runs its own batch of T tokens against its
own weight replica (tokens are independent: no collective in the step), so
`value` is N*T*K / max-rank time ("weak" scaling).

The JSON line also carries `workloads`: the decode, small and skewed40
workloads and the decode and prefill layers with FP8 gate/up projections
(moe_zc_forward_fp8, `dtype` says so) (--workloads), each timed the same way
in the same run, with its own ms_per_step, tokens/s, e2e,
roofline, layer_roofline and clocks (each timed region lasts at least about
a second, so the clocks are sampled inside it).
Also: `e2e` (the same metric through moe_zc_forward_host: the
step's input is copied from pinned host memory and its output back inside the
timed region, in chunks whose copies overlap the kernels), `roofline` (the dominant kernel's achieved rate against the measured
peak in MEASURED_PEAKS.json, from per-stage CUDA events recorded on the
forward's stream during a second timed region of K steps; the headline
region has no events between kernels, so they can overlap), `cpu_baseline` (the fp64 CPU oracle, as it stands, timed on the
host cores on a bounded token sample; rank 0, N=1 only), `clocks` (SM clocks
and throttle reasons sampled during the timed region) and `gpu_launches`.

--impl reference times the fp64 CPU oracle itself on the host cores (each
step a bounded token sample of the same workload) and prints the same line
with "impl": "reference".
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from mixture_experts_layer_28_b200 import workloads as wl  # noqa: E402

METRIC = "MoE-layer tokens/s; executed-FFN TFLOPS as % of B200 bf16 peak (HBM % at decode)"
UNIT = "tokens/s"
L2_BYTES = 126 * 2 ** 20


def kernels_per_forward(w, sms=148):
    """Kernels one forward launches (the library's own launch plan)."""
    from mixture_experts_layer_28_b200 import moe_zc as mz
    return mz.plan(w.T, w.d, w.N, w.Z, w.K, w.I, sms=sms, resident_blocks=sms)["kernels"]


# DRAM traffic of the dominant kernel: dram__bytes_read.sum +
# dram__bytes_write.sum of one launch over that launch's algorithmic bytes,
# from an ncu capture of a small case of the same kernel (the GEMM summaries
# under profiles/ give the command), with the sha256 (first 16 hex digits) of
# the GEMM engine's sources at the capture.  `traffic` = ratio x the
# algorithmic bytes of this run's launch (traffic scales with the units a
# launch processes); null when the sources have changed since the capture.
GEMM_SOURCES = ["gemm_tcgen05.cu", "ptx.cuh", "epilogue.cuh", "kernels.cuh", "step.cuh"]
NCU_TRAFFIC_RATIO = {
    # workload (+ "_fp8" for the FP8 forward): (dominant kernel,
    # DRAM bytes / algorithmic bytes, GEMM sources sha16, the captured case)
    "prefill": ("gateup_gemm", 3.5192e9 / 2.5460e9, "5becaa38c9c4f6e6",
                "T=8192, N=32, Z=16 prefill-shaped layer, ncu DRAM counters of two launches"),
    "prefill_fp8": ("gateup_gemm", 1.4575e9 / 1.4260e9, "5becaa38c9c4f6e6",
                    "T=8192, N=32, Z=16 prefill-shaped layer, ncu DRAM counters of two launches"),
    "decode": ("decode_step (route, dispatch, gate/up + down GEMMs, combine: one kernel)",
               1.4520e9 / 1.4687e9, "5becaa38c9c4f6e6",
               "T=64, N=32, Z=16 decode-shaped layer, ncu DRAM counters of two launches"),
    "decode_fp8": ("decode_step (route, dispatch, gate/up + down GEMMs, combine: one kernel)",
                   0.9802e9 / 0.9989e9, "5becaa38c9c4f6e6",
                   "T=64, N=32, Z=16 decode-shaped layer, ncu DRAM counters of two launches"),
}
SUSTAINED_REGION_S = 2.0   # timed regions at least this long use the sustained bf16 peak
NOMINAL_HBM_GBS = 7700.0   # B200 HBM3e, HGX figure (context beside the measured copy peak)
EXTRA_WORKLOADS = "decode,small,skewed40,decode_fp8,prefill_fp8"


def gemm_sources_sha16():
    import hashlib
    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        with open(os.path.join(ROOT, "mixture_experts_layer_28_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="prefill", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--chunk-tokens", type=int, default=0,
                    help="chunk size of the host-buffer forward (0: library default)")
    ap.add_argument("--graph", action="store_true",
                    help="time replays of one forward captured into a CUDA graph")
    ap.add_argument("--shape", default="",
                    help="override workload sizes, e.g. T=4096,N=32,Z=16 (for profiling runs)")
    ap.add_argument("--fp8", action="store_true",
                    help="time the forward with FP8 gate/up projections (moe_zc_forward_fp8)")
    ap.add_argument("--workloads", default=EXTRA_WORKLOADS,
                    help="comma-separated workloads also timed in the same run and reported "
                         "under `workloads` ('none': only the headline)")
    return ap.parse_args()


def workload_of(args) -> wl.Workload:
    kw = {}
    for item in filter(None, args.shape.split(",")):
        k, v = item.split("=")
        kw[k.strip()] = int(v)
    if kw:
        kw["name"] = f"{args.workload}[{args.shape}]"
    return wl.get(args.workload, **kw)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=p["hbm_gbs"], bf16=p["bf16_tflops"],
                    bf16_sus=p["bf16_tflops_sustained"], src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# ----------------------------------------------------------------- distributed
class Dist:
    def __init__(self, n_gpus: int):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        if self.world != n_gpus:
            raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={self.world}: launch N>1 with torchrun")
        self.pg = None
        self.cuda = torch.cuda.is_available()
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            if self.cuda:
                torch.cuda.set_device(self.local)
                dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                        device_id=torch.device("cuda", self.local))
            else:   # host-only ranks (tests of this plumbing)
                dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
            self.pg = dist
        elif self.cuda:
            torch.cuda.set_device(0)

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, v: float) -> float:
        """The largest v over all ranks (step times: the slowest rank sets the pace)."""
        if not self.pg:
            return v
        t = torch.tensor([v], dtype=torch.float64, device="cuda" if self.cuda else "cpu")
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples (every 100 ms, each with its own timestamp) of SM
    clocks and throttle reasons; summary() keeps the samples taken inside
    the timed region [t0, t1] (host wall clock)."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.5)
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return
        time.sleep(0.3)   # the sample covering the region's end
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)

    @staticmethod
    def _stamp(text):
        import datetime
        for fmt in ("%Y/%m/%d %H:%M:%S.%f", "%Y/%m/%d %H:%M:%S"):
            try:
                return datetime.datetime.strptime(text, fmt).timestamp()
            except ValueError:
                pass
        return None

    def summary(self, t0=None, t1=None):
        sm, mx, reasons, n_all = [], None, set(), 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 10:
                continue
            n_all += 1
            ts = self._stamp(parts[0])
            if t0 is not None and ts is not None and not (t0 - 0.1 <= ts <= t1 + 0.1):
                continue
            try:
                sm.append(float(parts[2]))
                mx = float(parts[3])
            except ValueError:
                continue
            for nm, v in zip(names, parts[6:10]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "samples_outside_region": n_all - len(sm)}


# ----------------------------------------------------------------- inputs
def make_inputs(w: wl.Workload):
    ri = wl.routing_inputs(w)
    b = ri.bias(w.N, w.delta)
    ew = wl.expert_weights(w, "cuda")
    dev = dict(x=ri.x.cuda(), W_r=ri.W_r.cuda(), b=b.cuda(),
               off=None if ri.logit_offset is None else ri.logit_offset.cuda())
    return ri, b, ew, dev


def routing_stats(w, cnt):
    ffn = cnt[: w.N].astype(np.int64)
    P = int(ffn.sum())
    hit = int((ffn > 0).sum())
    return dict(ffn_pairs=P, experts_hit=hit, zero_pick_fraction=1.0 - P / float(w.T * w.K),
                max_load=int(ffn.max()) if w.N else 0)


def roofline_numbers(w, st, pk, fp8=False, splits=1):
    """Algorithmic FLOPs and bytes of the layer and of its kernels.  fp8: the
    gate/up weights and permuted tokens are E4M3 bytes plus one scale byte
    per 32 elements; the down projection stays bf16.  splits: the router
    GEMM's K slices."""
    P, hit = st["ffn_pairs"], st["experts_hit"]
    d, I, T, E = w.d, w.I, w.T, w.E
    gu = (1.0 + 1.0 / 32) if fp8 else 2.0      # bytes per gate/up weight or token element
    F_gateup = 4.0 * d * I * P
    F_down = 2.0 * d * I * P
    B_gateup = hit * 2.0 * I * d * gu + P * d * gu + P * I * 2    # weights + Xp in + H out
    B_down = hit * 1.0 * I * d * 2 + P * I * 2 + P * d * 2        # weights + H in + Y out
    F_layer = F_gateup + F_down
    B_layer = hit * (2.0 * d * I * gu + d * I * 2) + E * d * 2 + E * 4 + 2.0 * T * d * 2
    # the rest of the forward, for a kernel that also routes, dispatches and
    # combines (the decode step's one grid): the router's K slices of partial
    # logits read; picks, gates, slots and zsum written; x read twice (copy
    # and combine), the permuted tokens written, Y read back, out written
    B_phases = (splits * T * E * 4 + T * w.K * 12 + T * 4 + 2.0 * T * d * 2 + P * d * gu
                + P * d * 2 + T * d * 2)
    return dict(F_gateup=F_gateup, F_down=F_down, B_gateup=B_gateup, B_down=B_down,
                F_layer=F_layer, B_layer=B_layer, B_phases=B_phases, fp8=fp8)


# ----------------------------------------------------------------- oracle timing
def oracle_sample_time(w, ri, b, ew, n_tokens, seed_offset=0):
    """Seconds the fp64 oracle takes for the forward of n sampled tokens.

    The weights of the experts those tokens pick are copied to host memory
    (bf16) before timing; widening them to fp64 is part of the oracle's work.
    """
    from oracle import moe_zc_ref as ref
    rows = wl.tokens_sample(w.T, n_tokens, w.seed + seed_offset)
    xs = ri.x[rows]
    r = ref.route(xs, ri.W_r, b, w.N, w.K, ri.logit_offset)
    hit = np.unique(r.idx[r.idx < w.N])
    host = {int(e): (ew.W_gate[e].cpu(), ew.W_up[e].cpu(), ew.W_down[e].cpu()) for e in hit}
    t0 = time.perf_counter()
    r = ref.route(xs, ri.W_r, b, w.N, w.K, ri.logit_offset)
    ref.forward_rows(xs, r, lambda e: host[e])
    return time.perf_counter() - t0, len(rows)


def cpu_baseline(w, ri, b, ew, target_s=12.0):
    """Oracle tokens/s on a seeded token sample grown until it takes about
    target_s of CPU time (or covers all T tokens).  The oracle's cost per
    token falls as more tokens share the widened expert weights, so the
    sample size is stated with the number."""
    cores = len(os.sched_getaffinity(0))
    n = min(w.T, 16)
    dt, n = oracle_sample_time(w, ri, b, ew, n, 1)
    for i in range(4):
        if dt >= target_s or n >= w.T:
            break
        n = int(min(w.T, max(2 * n, n * target_s / max(dt, 1e-3))))
        dt, n = oracle_sample_time(w, ri, b, ew, n, 2 + i)
    return {"value": n / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n} of {w.T} tokens (seeded sample), fp64 NumPy oracle, {dt:.1f} s"}


# ----------------------------------------------------------------- arms
def config_of(w, extra=None):
    c = {"workload": w.name, "T": w.T, "d": w.d, "N": w.N, "Z": w.Z, "K": w.K, "I": w.I,
         "target_zero_frac": w.zero_frac, "zipf_s": w.zipf_s, "seed": w.seed,
         "ffn_bias": "U[-0.1,0.1]" if w.bias == "random" else "0"}
    if extra:
        c.update(extra)
    return c


def bf16_peak(pk, region_s, clk=None):
    """The bf16 peak a kernel timed inside a region of region_s seconds is held
    to: the burst figure for a region under SUSTAINED_REGION_S, the sustained
    one (seconds of back-to-back GEMMs under the power cap) for a longer one.
    The clocks sampled in the region are reported beside the fraction, not
    used to pick the peak (the burst figure is the stricter one)."""
    if region_s >= SUSTAINED_REGION_S:
        return pk["bf16_sus"], f"bf16 dense, sustained ({pk['src']}, MEASURED_PEAKS.json)"
    return pk["bf16"], f"bf16 dense, burst ({pk['src']}, MEASURED_PEAKS.json)"


def tensor_peak(pk, region_s, clk=None, fp8=False):
    """bf16_peak, or for FP8 contractions that figure times 2 (the nominal
    dense FP8 / bf16 ratio of B200: 4.5 / 2.25 PFLOP/s)."""
    peak, kind = bf16_peak(pk, region_s, clk)
    if fp8:
        return 2.0 * peak, "FP8 dense = 2 x " + kind
    return peak, kind


def kernel_roofline(w, rf, plan, per, pk, region_s, clk=None):
    """The dominant stage's achieved rate against its bound."""
    dom = max(per, key=per.get)
    # (with the one-grid expert GEMMs the gate/up stage is the kernel that
    # runs both; with the decode step in that grid, also route, dispatch and
    # combine, whose bytes it then moves too)
    one_grid = bool(plan["expert_gemms_one_grid"])
    step = bool(plan.get("one_grid_step"))
    kern = {"gateup_gemm": ((rf["F_gateup"] + rf["F_down"],
                             rf["B_gateup"] + rf["B_down"] + (rf["B_phases"] if step else 0.0))
                            if one_grid else (rf["F_gateup"], rf["B_gateup"])),
            "down_gemm": (rf["F_down"], rf["B_down"])}.get(dom)
    if not kern or per[dom] <= 0:
        return None
    F, B = kern
    sec = per[dom] / 1e3
    # the FP8 forward's gate/up GEMM runs FP8 MMAs (its one-grid kernel also
    # the bf16 down tiles: held to the FP8 peak, the optimistic bound)
    peak, kind = tensor_peak(pk, region_s, clk, rf.get("fp8") and dom == "gateup_gemm")
    t_tensor, t_hbm = F / (peak * 1e12), B / (pk["hbm"] * 1e9)
    if t_tensor >= t_hbm:
        ach = F / sec / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                "frac": ach / peak, "peak_kind": kind,
                "frac_of_sustained_peak": ach / pk["bf16_sus"]}
    else:
        ach = B / sec / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": pk["hbm"], "unit": "GB/s",
                "frac": ach / pk["hbm"],
                "peak_kind": f"HBM copy, read + write ({pk['src']}, MEASURED_PEAKS.json)",
                "frac_of_nominal_hbm": ach / NOMINAL_HBM_GBS}
    roof["kernel"] = dom
    if one_grid and dom == "gateup_gemm":
        roof["kernel"] = ("decode_step (route, dispatch, gate/up + down GEMMs, combine: one kernel)"
                          if step else "gateup_down_gemm (one kernel)")
    roof["ms_per_launch"] = per[dom]
    roof["algorithmic_bytes"] = B
    roof["algorithmic_flops"] = F
    tr = NCU_TRAFFIC_RATIO.get(w.name + ("_fp8" if rf.get("fp8") else ""))
    roof["traffic"] = None
    if tr and tr[0] == roof["kernel"] and tr[2] == gemm_sources_sha16():
        roof["traffic"] = tr[1] * B
        roof["traffic_source"] = f"ncu DRAM bytes / algorithmic bytes = {tr[1]:.3f} on {tr[3]}"
    return roof


def layer_roofline(rf, pk, ms, region_s, clk=None):
    """The whole layer: the slower of executed FFN FLOPs at the tensor peak
    (FP8: the gate/up FLOPs at the FP8 peak, the down FLOPs at bf16) and the
    bytes it must touch at the HBM peak, against the measured step."""
    peak, kind = bf16_peak(pk, region_s, clk)
    if rf.get("fp8"):
        t_f = (rf["F_gateup"] / 2.0 + rf["F_down"]) / (peak * 1e12)
        kind = "gate/up at 2 x, down at 1 x " + kind
    else:
        t_f = rf["F_layer"] / (peak * 1e12)
    t_b = rf["B_layer"] / (pk["hbm"] * 1e9)
    sec = ms / 1e3
    ffn_tflops = rf["F_layer"] / sec / 1e12
    hbm_gbs = rf["B_layer"] / sec / 1e9
    return {"bound": "tensor" if t_f >= t_b else "hbm", "roofline_ms": max(t_f, t_b) * 1e3,
            "frac": max(t_f, t_b) / sec, "bf16_peak_kind": kind,
            "frac_vs_sustained_bf16": max(t_f * peak / pk["bf16_sus"], t_b) / sec,
            "executed_ffn_tflops": ffn_tflops,
            "pct_of_bf16_peak_burst": 100.0 * ffn_tflops / pk["bf16"],
            "pct_of_bf16_peak_sustained": 100.0 * ffn_tflops / pk["bf16_sus"],
            "hbm_gbs": hbm_gbs, "pct_of_hbm": 100.0 * hbm_gbs / pk["hbm"],
            "pct_of_nominal_hbm": 100.0 * hbm_gbs / NOMINAL_HBM_GBS}


def measure(args, dist, w, steps, e2e_steps, headline, fp8=False):
    """Time `steps` forwards of workload w (device-resident inputs), then the
    same with per-stage events, then e2e through the host-buffer entry point.
    steps <= 0: as many as fill about one second (at least 20).  fp8: the
    forward with FP8 gate/up (moe_zc_forward_fp8, e2e through
    moe_zc_forward_host_fp8; weights quantised on the device before
    timing)."""
    from mixture_experts_layer_28_b200 import moe_zc as mz
    pk = peaks()
    ri, b, ew, dev = make_inputs(w)
    out = torch.empty_like(dev["x"])
    stream = torch.cuda.current_stream()
    mz.reserve(w.T, w.d, w.N, w.Z, w.K, w.I)
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    plan = mz.plan(w.T, w.d, w.N, w.Z, w.K, w.I, sms=sms, resident_blocks=sms)
    if fp8:
        q_gate, q_up = mz.fp8_quantize_weights(ew.W_gate), mz.fp8_quantize_weights(ew.W_up)
        torch.cuda.synchronize()

    def step(x=None, o=None):
        if fp8:
            mz.forward_fp8(dev["x"] if x is None else x, dev["W_r"], dev["b"], q_gate, q_up,
                           ew.W_down, w.N, w.Z, w.K, out=out if o is None else o,
                           logit_offset=dev["off"], stream=stream)
            return
        mz.forward(dev["x"] if x is None else x, dev["W_r"], dev["b"], ew.W_gate, ew.W_up,
                   ew.W_down, w.N, w.Z, w.K, out=out if o is None else o,
                   logit_offset=dev["off"], stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    mz.synchronize()
    st = routing_stats(w, mz.expert_load(w.E))
    rf = roofline_numbers(w, st, pk, fp8=fp8, splits=plan["router_k_slices"])
    if steps <= 0:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(5):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        steps = max(20, int(1.0 / max(e0.elapsed_time(e1) / 5 / 1e3, 1e-6)))
        steps = int(dist.max(float(steps)))   # every rank the same count

    # --graph: the forward captured once into a CUDA graph (its launches on
    # the capture stream), each timed step one replay
    graph = None
    if args.graph and headline:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            mz.forward(dev["x"], dev["W_r"], dev["b"], ew.W_gate, ew.W_up, ew.W_down,
                       w.N, w.Z, w.K, out=out, logit_offset=dev["off"])
        for _ in range(args.warmup):
            graph.replay()
        torch.cuda.synchronize()

    def timed_step():
        if graph is not None:
            graph.replay()
        else:
            step()

    # ---- device-resident timed region (no per-stage events: they would
    # separate the kernels and undo the overlap of dependent launches)
    clocks = ClockSampler(dist.local) if dist.rank == 0 else None
    if clocks:
        clocks.start()
    dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.time()
    e0.record(stream)
    for _ in range(steps):
        timed_step()
    e1.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    dist.barrier()
    ms = e0.elapsed_time(e1) / steps
    clk = None
    if clocks:
        clocks.stop()
        clk = clocks.summary(t0, t1)
    mz.synchronize()
    ms_max = dist.max(ms)
    region_s = ms_max * steps / 1e3
    value = dist.world * w.T / (ms_max / 1e3)

    # ---- a second timed region of the same length with CUDA events between
    # the forward's kernels on its stream: per-stage times for the roofline
    mz.profile(True)
    dist.barrier()
    torch.cuda.synchronize()
    n_prof = min(steps, 256)
    for _ in range(n_prof):
        step()
    torch.cuda.synchronize()
    dist.barrier()
    stage_ms, nfw = mz.profile_read()
    mz.profile(False)
    mz.synchronize()

    # ---- end to end through the host-buffer entry point: the step's input
    # goes from pinned host memory to the device and its output comes back,
    # in chunks whose copies overlap the kernels (moe_zc_forward_host)
    x_host = ri.x.pin_memory()
    out_host = torch.empty_like(x_host).pin_memory()

    def step_host():
        if fp8:
            mz.forward_host_fp8(x_host, dev["W_r"], dev["b"], q_gate, q_up, ew.W_down,
                                w.N, w.Z, w.K, out_host=out_host, logit_offset=dev["off"],
                                chunk_tokens=args.chunk_tokens, stream=stream)
            return
        mz.forward_host(x_host, dev["W_r"], dev["b"], ew.W_gate, ew.W_up, ew.W_down,
                        w.N, w.Z, w.K, out_host=out_host, logit_offset=dev["off"],
                        chunk_tokens=args.chunk_tokens, stream=stream)

    e2e_ms = None
    if e2e_steps > 0:
        for _ in range(2):
            step_host()
        torch.cuda.synchronize()
        dist.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(e2e_steps):
            step_host()
        e1.record(stream)
        torch.cuda.synchronize()
        dist.barrier()
        e2e_ms = dist.max(e0.elapsed_time(e1) / e2e_steps)
        mz.synchronize()

    per = {k: v / max(nfw, 1) for k, v in stage_ms.items()}
    res = {
        "value": value, "ms_per_step": ms_max, "steps": steps,
        "e2e": None if e2e_ms is None else {
            "value": dist.world * w.T / (e2e_ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": int(x_host.numel() * 2),
            "d2h_bytes_per_step": int(out_host.numel() * 2), "ms_per_step": e2e_ms,
            "steps": e2e_steps},
        "roofline": kernel_roofline(w, rf, plan, per, pk, region_s, clk),
        "layer_roofline": layer_roofline(rf, pk, ms_max, region_s, clk),
        "gpu_launches": plan["kernels"] * steps,
        "clocks": clk,
        "routing": st,
        "stage_ms": {k: round(v, 5) for k, v in per.items()},
        "touched_bytes": st["experts_hit"] * 3.0 * w.d * w.I * 2,
        "_keep": (ri, b, ew),
    }
    del graph
    return res


def run_ours(args, dist, w):
    res = measure(args, dist, w, args.steps, args.e2e_steps, headline=True, fp8=args.fp8)
    ri, b, ew = res.pop("_keep")
    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, ri, b, ew)
    del ri, b, ew
    touched = res.pop("touched_bytes")
    line = {
        "metric": METRIC, "value": res["value"], "unit": UNIT, "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8 gate/up (E4M3, 1x32 UE8M0 blocks), bf16 down" if args.fp8 else "bf16",
        "data": "synthetic: seeded inputs, random-init weights of the workload's shapes",
        "config": config_of(w, {
            "global_batch": w.T * dist.world, "parallelism": f"replicas{dist.world}",
            "cuda_graph": bool(args.graph),
            "l2": f"no flush: expert weights touched per step {touched / 1e9:.2f} GB > L2 126 MB"}),
        "e2e": res["e2e"],
        "roofline": res["roofline"],
        "layer_roofline": res["layer_roofline"],
        "cpu_baseline": cpu,
        "gpu_launches": res["gpu_launches"],
        "clocks": res["clocks"],
        "routing": res["routing"],
        "stage_ms": res["stage_ms"],
    }
    extra = [n for n in args.workloads.split(",") if n and n != "none" and n != w.name]
    if extra:
        line["workloads"] = {}
    for name in extra:
        gc_collect()
        fp8 = name.endswith("_fp8")
        wx = wl.get(name[:-4] if fp8 else name)
        r = measure(args, dist, wx, 0, max(args.e2e_steps, 20), headline=False, fp8=fp8)
        r.pop("_keep")
        touched = r.pop("touched_bytes")
        r["dtype"] = "fp8 gate/up (E4M3, 1x32 UE8M0 blocks), bf16 down" if fp8 else "bf16"
        r["config"] = config_of(wx, {
            "global_batch": wx.T * dist.world,
            "l2": (f"no flush: expert weights touched per step {touched / 1e9:.2f} GB"
                   f"{' > ' if touched > L2_BYTES else ' <= '}L2 126 MB")})
        line["workloads"][name] = r
    return line


def gc_collect():
    import gc
    gc.collect()
    torch.cuda.empty_cache()


def run_reference(args, dist, w):
    """The fp64 CPU oracle, as it stands, on the host cores."""
    if dist.rank != 0:
        return None
    ri = wl.routing_inputs(w)
    b = ri.bias(w.N, w.delta)
    ew = wl.expert_weights(w, "cuda" if torch.cuda.is_available() else "cpu")
    cores = len(os.sched_getaffinity(0))
    # Size the per-step sample so the whole run stays within about two
    # minutes: grow it from 16 tokens (doubling, then scaling) while a step
    # takes under the per-step share; the oracle's cost per token falls as
    # more tokens share the widened expert weights, so a probe of a few
    # tokens would overstate it.
    per_step = 120.0 / max(args.steps + args.warmup, 1)
    n = min(w.T, 16)
    dt, n = oracle_sample_time(w, ri, b, ew, n, 100)
    for i in range(8):
        if dt >= 0.5 * per_step or n >= w.T:
            break
        n = int(min(w.T, max(2 * n, n * 0.8 * per_step / max(dt, 1e-3))))
        dt, n = oracle_sample_time(w, ri, b, ew, n, 101 + i)
    for i in range(args.warmup):
        oracle_sample_time(w, ri, b, ew, n, 200 + i)
    tot = 0.0
    for i in range(args.steps):
        dt, n = oracle_sample_time(w, ri, b, ew, n, 300 + i)
        tot += dt
    ms = tot / args.steps * 1e3
    value = n / (ms / 1e3)
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic: seeded inputs, random-init weights of the workload's shapes",
        "config": config_of(w, {"global_batch": w.T, "parallelism": "cpu"}),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{n} of {w.T} tokens per step (seeded samples), fp64 NumPy oracle"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    w = workload_of(args)
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return
        line = run_reference(args, Dist(1) if int(os.environ.get("WORLD_SIZE", "1")) == 1 else _Rank0(args.gpus), w)
        print(json.dumps(line), flush=True)
        return
    dist = Dist(args.gpus)
    try:
        line = run_ours(args, dist, w)
        if dist.rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        dist.close()


class _Rank0:
    """Rank 0 of a torchrun launch of the reference arm: works alone."""

    def __init__(self, n):
        self.world, self.rank, self.local = n, 0, 0


if __name__ == "__main__":
    main()
