"""Find the zero-expert bias shift `delta` of each workload with the fp64 router.

TEST INFRASTRUCTURE: calls only the oracle and the seeded input generators.

A workload asks that a stated share of all T*K picks land on zero experts
("b set so ~30% of picks are zero experts").  With b = b0 + delta on the zero
experts, that share can only grow with delta (raising a zero expert's score
never pushes another zero expert out), so bisection on delta finds it.  The
shifts are written to mixture_experts_layer_28_b200/bias_shift.json, which
the input generators read.

    python -m oracle.calibrate_bias_shift [workload ...]
"""
from __future__ import annotations

import json
import os
import sys

import numpy as np

from mixture_experts_layer_28_b200 import workloads as wl
from oracle import moe_zc_ref
from oracle.moe_zc_ref import router_logits, softmax, _f64

OUT = os.path.join(os.path.dirname(wl.__file__), "bias_shift.json")
TOL = 0.005


def zero_share(p: np.ndarray, b0: np.ndarray, N: int, K: int, delta: float) -> float:
    """Share of all T*K picks that land on zero experts when every zero
    expert's bias is shifted by delta.

    The picks are the oracle's own: the top-K of s = p + b (bias added after
    the softmax, equal scores to the lower index, so an FFN expert wins a tie
    against a zero expert), counted with zero_pick_fraction.
    """
    s = p + b0[None, :]
    s[:, N:] += delta
    idx, _ = moe_zc_ref.select_topk(s, K)
    return moe_zc_ref.zero_pick_fraction(idx, N)


def calibrate(w: wl.Workload) -> float:
    ri = wl.routing_inputs(w)
    p = softmax(router_logits(ri.x, ri.W_r, ri.logit_offset))
    b0 = _f64(ri.b0)
    lo, hi = -1.0, 1.0
    for _ in range(60):
        mid = 0.5 * (lo + hi)
        f = zero_share(p, b0, w.N, w.K, mid)
        if abs(f - w.zero_frac) <= TOL / 4:
            return mid
        if f < w.zero_frac:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def main(names):
    data = {}
    if os.path.exists(OUT):
        with open(OUT) as f:
            data = json.load(f)
    for name in names:
        w = wl.WORKLOADS[name]
        if w.zero_frac is None:
            continue
        delta = calibrate(w)
        data[name] = delta
        print(f"{name}: delta = {delta!r}", flush=True)
    with open(OUT, "w") as f:
        json.dump(data, f, indent=1, sort_keys=True)
        f.write("\n")


if __name__ == "__main__":
    main(sys.argv[1:] or [n for n, w in wl.WORKLOADS.items() if w.zero_frac is not None])
