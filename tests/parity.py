"""Helpers of the GPU parity tests: run the CUDA path through the C ABI, run
the fp64 oracle on the same seeded inputs, and compare.

Tolerances:
  * routing -- bit-exact expert sets and an exact histogram on every token
    whose K-th and (K+1)-th biased scores (fp64 oracle) differ by at least
    TIE = 1e-5; for the rest (near-ties, where both choices are correct) the
    GPU's picks must be a valid top-K within TIE.  Gates: rtol 1e-4.  A
    gate's relative error is about its logit's absolute error (softmax), and
    the logits are fp32 sums of d bf16 products accumulated by the tensor
    cores (d = 6144: ~2e-5 measured).  That is far below what could move a
    pick: s = p + b with p ~ 1e-3 moves by ~1e-8, against the 1e-5 margin.
  * output -- the contract max|err| <= 2e-2 (1 + |ref|), and, because that
    bound is loose at these magnitudes (|out| ~ 1e-2..1), also
    |err| <= 5u (|ref| + rms(ref)) elementwise, u = 2^-8 the unit roundoff of
    bf16: the GPU rounds out once (<= u |ref|) and each FFN term carries the
    bf16 rounding of H and Y (a few u of the term, whose size is set by
    rms(ref)).  Measured: the GPU's max error equals that of rounding the
    exact result to bf16 alone; the worst element reaches ~2.6u.
  * per-expert H rows -- |err| <= 2u (|ref| + rms(ref)) (one bf16 rounding);
    Y rows -- |err| <= 4u (|ref| + rms(ref)) (Y's rounding plus H's rounding
    carried through W_down).
"""
from __future__ import annotations

import numpy as np
import torch

from mixture_experts_layer_28_b200 import moe_zc as mz
from mixture_experts_layer_28_b200 import workloads as wl
from oracle import moe_zc_ref as ref

TIE = 1e-5
U = 2.0 ** -8          # unit roundoff of bf16


class Case:
    """Inputs of one forward, on the host and on the device."""

    def __init__(self, w: wl.Workload, T=None, bias=None, weights_device="cuda"):
        self.w = w
        ri = wl.routing_inputs(w, T)
        self.T = ri.x.shape[0]
        self.x, self.W_r, self.off = ri.x, ri.W_r, ri.logit_offset
        self.b = ri.bias(w.N, w.delta) if bias is None else bias.to(torch.float32)
        self.ew = wl.expert_weights(w, weights_device) if w.N > 0 else None
        self.dev = dict(
            x=self.x.cuda(), W_r=self.W_r.cuda(), b=self.b.cuda(),
            off=None if self.off is None else self.off.cuda())

    def run(self, out=None, stream=None):
        w, d = self.w, self.dev
        ew = self.ew
        return mz.forward(d["x"], d["W_r"], d["b"],
                          ew.W_gate if ew else None, ew.W_up if ew else None,
                          ew.W_down if ew else None, w.N, w.Z, w.K, out=out,
                          logit_offset=d["off"], stream=stream)

    def expert(self, e):
        ew = self.ew
        return (ew.W_gate[e].double().cpu().numpy(), ew.W_up[e].double().cpu().numpy(),
                ew.W_down[e].double().cpu().numpy())

    def oracle_routing(self, rows=None):
        x = self.x if rows is None else self.x[rows]
        return ref.route(x, self.W_r, self.b, self.w.N, self.w.K, self.off)


def check_routing(case: Case, r: ref.Routing, idx_g, gate_g, cnt_g):
    """Exact routing and histogram away from near-ties; valid picks at them."""
    w = case.w
    N, K, E = w.N, w.K, w.E
    near = r.gap < TIE
    ok = ~near
    # GPU order: K distinct experts, largest score first
    assert all(len(set(row)) == K for row in idx_g.tolist())
    so, sg = np.sort(r.idx, axis=1), np.sort(idx_g, axis=1)
    bad = np.nonzero((so != sg).any(axis=1) & ok)[0]
    assert bad.size == 0, f"{bad.size} tokens route differently, first {bad[:5]}"
    # gates, matched by expert
    og = np.take_along_axis(r.gate, np.argsort(r.idx, 1), 1)
    gg = np.take_along_axis(gate_g.astype(np.float64), np.argsort(idx_g, 1), 1)
    np.testing.assert_allclose(gg[ok], og[ok], rtol=1e-4, atol=1e-9)
    # histogram: exact against the GPU's own picks, and against the oracle
    # once near-tie tokens are taken out of both
    assert np.array_equal(cnt_g, np.bincount(idx_g.ravel(), minlength=E))
    cg = cnt_g - np.bincount(idx_g[near].ravel(), minlength=E)
    co = ref.expert_load(r.idx, E) - np.bincount(r.idx[near].ravel(), minlength=E)
    assert np.array_equal(cg, co)
    # near-ties: the GPU's picks are a top-K within the tie margin
    s = r.p + np.asarray(case.b, dtype=np.float64)[None, :]
    for t in np.nonzero(near)[0]:
        S = idx_g[t]
        rest = np.setdiff1d(np.arange(E), S)
        if rest.size:
            assert s[t, S].min() >= s[t, rest].max() - TIE
    return ok


def check_output(out_g: np.ndarray, out_o: np.ndarray):
    err = np.abs(out_g - out_o)
    bound = 2e-2 * (1.0 + np.abs(out_o))
    assert np.all(err <= bound), f"contract bound broken: max excess {(err - bound).max()}"
    rms = float(np.sqrt(np.mean(out_o ** 2)))
    ratio = err / (np.abs(out_o) + rms)
    assert ratio.max() <= 5 * U, f"max|err|/(|ref|+rms) = {ratio.max():.3e} > 5u"
    return float(err.max()), rms


def check_expert_rows(case: Case, e: int, max_rows=64):
    """H and Y rows of FFN expert e (from moe_zc_last_expert) against fp64."""
    w = case.w
    tok, Hg, Yg, n = mz.last_expert(e, w.d, w.I, max_rows)
    if n == 0:
        return 0
    Wg, Wu, Wd = case.expert(e)
    xs = case.x[torch.from_numpy(tok.astype(np.int64))].double().numpy()
    a = xs @ Wg.T
    Ho = ref.silu(a) * (xs @ Wu.T)
    Yo = Ho @ Wd.T
    for g, o, name, k in ((Hg.double().numpy(), Ho, "H", 2), (Yg.double().numpy(), Yo, "Y", 4)):
        rms = float(np.sqrt(np.mean(o ** 2)))
        ratio = np.abs(g - o) / (np.abs(o) + rms)
        assert ratio.max() <= k * U, f"expert {e} {name}: max err/(|ref|+rms) {ratio.max():.3e}"
    return n
