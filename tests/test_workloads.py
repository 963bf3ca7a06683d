"""Seeded inputs: determinism, shapes, and the calibrated zero-expert share."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_28_b200 import workloads as wl
from oracle import moe_zc_ref as ref


def test_routing_inputs_deterministic_and_shaped():
    w = wl.get("tiny")
    a, b = wl.routing_inputs(w), wl.routing_inputs(w)
    assert torch.equal(a.x, b.x) and torch.equal(a.W_r, b.W_r) and torch.equal(a.b0, b.b0)
    assert a.x.shape == (w.T, w.d) and a.x.dtype == torch.bfloat16
    assert a.W_r.shape == (w.E, w.d) and a.W_r.dtype == torch.bfloat16
    assert a.b0.dtype == torch.float32 and float(a.b0.abs().max()) <= 0.1
    assert abs(float(a.x.float().std()) - 1.0) < 0.02
    assert abs(float(a.W_r.float().std()) - w.w_std) < 0.1 * w.w_std


def test_prefix_tokens_match():
    w = wl.get("small")
    full, part = wl.routing_inputs(w), wl.routing_inputs(w, T=100)
    assert torch.equal(full.x[:100], part.x)


def test_expert_weights_cpu():
    w = wl.get("tiny")
    ew = wl.expert_weights(w)
    assert ew.W_gate.shape == (w.N, w.I, w.d)
    assert ew.W_down.shape == (w.N, w.d, w.I)
    assert abs(float(ew.W_up.float().std()) - w.w_std) < 0.05 * w.w_std
    assert torch.equal(ew.W_gate, wl.expert_weights(w).W_gate)


def test_zipf_offset():
    w = wl.get("skewed40")
    ri = wl.routing_inputs(w)
    off = ri.logit_offset
    assert off is not None and torch.all(off[w.N:] == 0)
    ranks = torch.exp(-off[: w.N].double() / w.zipf_s).round().long().sort().values
    assert torch.equal(ranks, torch.arange(1, w.N + 1))


@pytest.mark.slow
@pytest.mark.parametrize("name", ["prefill", "decode", "skewed20", "skewed40", "skewed60",
                                  "prefill_balanced", "decode_balanced"])
def test_calibrated_zero_share(name):
    """The stored bias shift gives the workload's zero-expert share (fp64 router)."""
    w = wl.get(name)
    ri = wl.routing_inputs(w)
    r = ref.route(ri.x, ri.W_r, ri.bias(w.N, w.delta), w.N, w.K, ri.logit_offset)
    assert abs(ref.zero_pick_fraction(r.idx, w.N) - w.zero_frac) <= 0.005


def test_balanced_companions_share_x_and_router():
    """The balanced workloads differ from their LongCat-shaped twins only in b:
    same x and W_r, FFN bias zero, and one shift on the zero experts."""
    for name in ["prefill", "decode"]:
        w, wb = wl.get(name, T=32), wl.get(name + "_balanced", T=32)
        a, b = wl.routing_inputs(w), wl.routing_inputs(wb)
        assert torch.equal(a.x, b.x) and torch.equal(a.W_r, b.W_r)
        bb = b.bias(wb.N, wb.delta)
        assert torch.all(bb[: wb.N] == 0) and torch.all(bb[wb.N:] == wb.delta)


@pytest.mark.slow
def test_balanced_prefill_spreads_load():
    """With no FFN bias every FFN expert is hit and none takes more than a
    few times the mean load (fp64 router)."""
    w = wl.get("prefill_balanced")
    ri = wl.routing_inputs(w)
    r = ref.route(ri.x, ri.W_r, ri.bias(w.N, w.delta), w.N, w.K)
    ffn = ref.expert_load(r.idx, w.E)[: w.N]
    assert (ffn > 0).all() and ffn.max() < 2 * ffn.mean()
