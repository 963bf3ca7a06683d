"""Plant plausible mistakes in the oracle and check that some pin catches each.

Every mutant below breaks one reading of the LongCat-Flash write-up's
"Zero-computation experts" section (softmax over all experts, bias for
selection only, unbiased gates, identity zero experts, SwiGLU experts,
lower-index ties, histogram over all experts, zero experts at indices
N..E-1), or of the helpers that measure and calibrate the zero-expert share
of the picks (the workloads' "b set so ~X% of picks are zero experts").  A mutant that no pin catches
would mean the oracle could carry that mistake unnoticed.
"""
import numpy as np
import pytest

from oracle import calibrate_bias_shift as cal
from oracle import moe_zc_ref as ref
from oracle_pins import ALL_PINS

_orig = {k: getattr(ref, k) for k in ("softmax", "select_topk", "route", "silu",
                                      "swiglu_expert", "forward_rows", "expert_load",
                                      "router_logits", "zero_pick_fraction")}
_orig_cal = {"zero_share": cal.zero_share}


def _route_bias_before_softmax(x, W_r, b, N, K, logit_offset=None):
    l = ref.router_logits(x, W_r, logit_offset) + ref._f64(b)[None, :]
    p = ref.softmax(l)
    idx, gap = ref.select_topk(p, K)
    return ref.Routing(idx=idx, gate=np.take_along_axis(p, idx, 1), gap=gap, p=p, N=N)


def _route_renormalised(x, W_r, b, N, K, logit_offset=None):
    r = _orig["route"](x, W_r, b, N, K, logit_offset)
    r.gate = r.gate / r.gate.sum(axis=1, keepdims=True)
    return r


def _route_gate_biased(x, W_r, b, N, K, logit_offset=None):
    r = _orig["route"](x, W_r, b, N, K, logit_offset)
    r.gate = r.gate + ref._f64(b)[r.idx]
    return r


def _route_softmax_ffn_only(x, W_r, b, N, K, logit_offset=None):
    l = ref.router_logits(x, W_r, logit_offset)
    p = np.zeros_like(l)
    p[:, :N] = ref.softmax(l[:, :N])
    p[:, N:] = np.exp(l[:, N:] - l.max(axis=1, keepdims=True))
    s = p + ref._f64(b)[None, :]
    idx, gap = ref.select_topk(s, K)
    return ref.Routing(idx=idx, gate=np.take_along_axis(p, idx, 1), gap=gap, p=p, N=N)


def _topk_smallest(s, K):
    return _orig["select_topk"](-s, K)


def _topk_ties_high(s, K):
    E = s.shape[1]
    idx, gap = _orig["select_topk"](s[:, ::-1], K)
    return E - 1 - idx, gap


def _softmax_no_norm(l):
    return np.exp(l - l.max(axis=1, keepdims=True))


def _silu_wrong_sign(z):
    return z / (1.0 + np.exp(z))


def _swiglu_gate_up_swapped(xs, Wg, Wu, Wd):
    return _orig["swiglu_expert"](xs, Wu, Wg, Wd)


def _swiglu_no_silu(xs, Wg, Wu, Wd):
    xs = ref._f64(xs)
    return ((xs @ ref._f64(Wg).T) * (xs @ ref._f64(Wu).T)) @ ref._f64(Wd).T


def _swiglu_down_rows_reversed(xs, Wg, Wu, Wd):
    xs = ref._f64(xs)
    h = ref.silu(xs @ ref._f64(Wg).T) * (xs @ ref._f64(Wu).T)
    return h @ ref._f64(Wd)[::-1].T


def _forward_rows_drop_zero(x, r, expert):
    out = _orig["forward_rows"](x, r, expert)
    return out - r.zsum[:, None] * ref._f64(x)


def _forward_rows_zero_is_zero_gate(x, r, expert):
    out = _orig["forward_rows"](x, r, expert)
    return out - r.zsum[:, None] * ref._f64(x) + r.zsum.mean() * ref._f64(x)


def _load_drops_last_expert(idx, E):
    c = _orig["expert_load"](idx, E)
    c[E - 1] = 0
    return c


def _logits_offset_negated(x, W_r, logit_offset=None):
    l = ref._f64(x) @ ref._f64(W_r).T
    if logit_offset is not None:
        l = l - ref._f64(logit_offset)[None, :]
    return l


def _zero_fraction_strict(idx, N):
    idx = np.asarray(idx)
    return float((idx > N).sum()) / max(idx.size, 1)


def _zero_fraction_counts_last_ffn(idx, N):
    idx = np.asarray(idx)
    return float((idx >= N - 1).sum()) / max(idx.size, 1)


def _zero_share_ties_to_zero(p, b0, N, K, delta):
    # every zero expert scoring at least the K-th score counts, so a tie at
    # the selection boundary goes to the zero expert (and can exceed K picks)
    s = p + b0[None, :]
    s[:, N:] += delta
    T, E = s.shape
    if K >= E:
        return (E - N) / E
    kth = -np.partition(-s, K - 1, axis=1)[:, K - 1]
    return float((s[:, N:] >= kth[:, None]).sum()) / (T * K)


def _zero_share_shifts_ffn(p, b0, N, K, delta):
    s = p + b0[None, :]
    s[:, :N] += delta
    idx, _ = ref.select_topk(s, K)
    return ref.zero_pick_fraction(idx, N)


def _zero_share_strict_boundary(p, b0, N, K, delta):
    s = p + b0[None, :]
    s[:, N:] += delta
    idx, _ = ref.select_topk(s, K)
    return float((idx > N).sum()) / idx.size


MUTANTS = {
    "bias_before_softmax": ("route", _route_bias_before_softmax),
    "renormalised_gates": ("route", _route_renormalised),
    "gate_includes_bias": ("route", _route_gate_biased),
    "softmax_over_ffn_only": ("route", _route_softmax_ffn_only),
    "topk_smallest": ("select_topk", _topk_smallest),
    "ties_to_higher_index": ("select_topk", _topk_ties_high),
    "softmax_not_normalised": ("softmax", _softmax_no_norm),
    "silu_wrong_sign": ("silu", _silu_wrong_sign),
    "gate_up_swapped": ("swiglu_expert", _swiglu_gate_up_swapped),
    "no_silu": ("swiglu_expert", _swiglu_no_silu),
    "down_rows_reversed": ("swiglu_expert", _swiglu_down_rows_reversed),
    "zero_expert_dropped": ("forward_rows", _forward_rows_drop_zero),
    "zero_expert_wrong_gate": ("forward_rows", _forward_rows_zero_is_zero_gate),
    "load_drops_last_zero_expert": ("expert_load", _load_drops_last_expert),
    "offset_sign_flipped": ("router_logits", _logits_offset_negated),
    "zero_fraction_misses_expert_N": ("zero_pick_fraction", _zero_fraction_strict),
    "zero_fraction_counts_last_ffn": ("zero_pick_fraction", _zero_fraction_counts_last_ffn),
    "zero_share_ties_to_zero_expert": ("cal.zero_share", _zero_share_ties_to_zero),
    "zero_share_shifts_ffn_bias": ("cal.zero_share", _zero_share_shifts_ffn),
    "zero_share_misses_expert_N": ("cal.zero_share", _zero_share_strict_boundary),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    if attr.startswith("cal."):
        monkeypatch.setattr(cal, attr[4:], fn)
    else:
        monkeypatch.setattr(ref, attr, fn)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(ref)
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"mutant {name} passed every pin"
