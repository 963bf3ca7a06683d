"""Checks that pin the fp64 oracle to things other than itself.

Each ``pin_*`` takes the oracle module (``oracle.moe_zc_ref``) and raises
AssertionError when the oracle disagrees with what the LongCat-Flash write-up
and plain mathematics fix: hand-solved worked examples, brute force over all
K-subsets, pure-Python scalar loops, closed forms for the special cases, a
textbook softmax-top-K MoE written with torch, and invariants.  They are
collected by test_oracle_pins.py, and test_oracle_mutants.py plants plausible
mistakes in the oracle to show that each one is caught by some pin.
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _layer(seed, T, d, N, Z, I, w_std=0.3, b_scale=0.1):
    r = _rng(seed)
    E = N + Z
    return dict(
        x=r.standard_normal((T, d)),
        W_r=r.standard_normal((E, d)) * w_std,
        b=r.uniform(-b_scale, b_scale, E),
        W_gate=r.standard_normal((N, I, d)) * w_std,
        W_up=r.standard_normal((N, I, d)) * w_std,
        W_down=r.standard_normal((N, d, I)) * w_std,
    )


def _fwd(ref, L, N, Z, K, **kw):
    return ref.forward(L["x"], L["W_r"], L["b"], L["W_gate"], L["W_up"], L["W_down"],
                       N, Z, K, **kw)


# ---------------------------------------------------------------------------
def pin_worked_examples(ref):
    """Hand-solved tiny layers (tests/golden/worked_examples.json)."""
    with open(os.path.join(GOLDEN, "worked_examples.json")) as f:
        data = json.load(f)
    for ex in data["examples"]:
        N, Z, K = ex["N"], ex["Z"], ex["K"]
        W = {k: np.array(ex[k], dtype=np.float64) for k in ("x", "W_r", "b", "W_gate", "W_up", "W_down")}
        out, r = ref.forward(W["x"], W["W_r"], W["b"], W["W_gate"], W["W_up"], W["W_down"], N, Z, K)
        for t in range(len(ex["x"])):
            got = sorted(int(i) for i in r.idx[t])
            assert got == ex["expected_idx_set"][t], (ex["name"], got)
            gmap = {int(i): float(g) for i, g in zip(r.idx[t], r.gate[t])}
            want = dict(zip(ex["expected_idx_set"][t], ex["expected_gate"][t]))
            for i in want:
                assert abs(gmap[i] - want[i]) <= 1e-12, (ex["name"], i)
        np.testing.assert_allclose(out, np.array(ex["expected_out"]), rtol=1e-12, atol=1e-12,
                                   err_msg=ex["name"])
        load = ref.expert_load(r.idx, N + Z)
        assert load.tolist() == ex["expected_load"], (ex["name"], load)


def pin_topk_brute_force(ref):
    """Top-K equals the K-subset with the largest score sum (all subsets tried)."""
    r = _rng(1)
    for E, K in [(4, 1), (5, 2), (7, 3), (12, 3), (9, 4)]:
        s = r.uniform(-1, 1, (40, E))
        idx, gap = ref.select_topk(s, K)
        for t in range(s.shape[0]):
            best = max(itertools.combinations(range(E), K), key=lambda c: sum(s[t, list(c)]))
            assert sorted(idx[t].tolist()) == list(best), (E, K, t)
            srt = np.sort(s[t])[::-1]
            assert abs(gap[t] - (srt[K - 1] - srt[K])) <= 1e-15
        # largest score first
        assert np.all(np.diff(np.take_along_axis(s, idx, 1), axis=1) <= 0)


def pin_topk_ties_lower_index(ref):
    """With exact ties, the lexicographically smallest best subset is chosen."""
    r = _rng(2)
    for E, K in [(6, 2), (8, 3), (10, 4)]:
        s = r.integers(0, 3, (60, E)).astype(np.float64)   # many exact ties
        idx, gap = ref.select_topk(s, K)
        for t in range(s.shape[0]):
            best_sum = max(sum(s[t, list(c)]) for c in itertools.combinations(range(E), K))
            cands = [c for c in itertools.combinations(range(E), K) if sum(s[t, list(c)]) == best_sum]
            assert sorted(idx[t].tolist()) == list(min(cands)), (E, K, t, s[t])
            assert gap[t] >= 0


def _py_softmax(l):
    m = max(l)
    e = [math.exp(v - m) for v in l]
    z = sum(e)
    return [v / z for v in e]


def _py_expert(x, Wg, Wu, Wd):
    I, d = len(Wg), len(x)
    h = []
    for i in range(I):
        a = sum(Wg[i][k] * x[k] for k in range(d))
        u = sum(Wu[i][k] * x[k] for k in range(d))
        h.append(a / (1.0 + math.exp(-a)) * u)
    return [sum(Wd[j][i] * h[i] for i in range(I)) for j in range(d)]


def pin_scalar_loops(ref):
    """The whole layer in pure-Python scalar loops on a few tokens."""
    N, Z, K, d, I = 3, 2, 2, 5, 4
    L = _layer(3, T=6, d=d, N=N, Z=Z, I=I)
    out, r = _fwd(ref, L, N, Z, K)
    xl, Wr, b = L["x"].tolist(), L["W_r"].tolist(), L["b"].tolist()
    Wg, Wu, Wd = L["W_gate"].tolist(), L["W_up"].tolist(), L["W_down"].tolist()
    for t, x in enumerate(xl):
        logits = [sum(Wr[e][k] * x[k] for k in range(d)) for e in range(N + Z)]
        p = _py_softmax(logits)
        s = [p[e] + b[e] for e in range(N + Z)]
        picks = sorted(range(N + Z), key=lambda e: (-s[e], e))[:K]
        assert sorted(picks) == sorted(r.idx[t].tolist())
        o = [0.0] * d
        for e in picks:
            y = x if e >= N else _py_expert(x, Wg[e], Wu[e], Wd[e])
            o = [o[j] + p[e] * y[j] for j in range(d)]
        np.testing.assert_allclose(out[t], o, rtol=1e-12, atol=1e-13)


def pin_single_expert_is_swiglu(ref):
    """N=1, Z=0, K=1: the gate is 1 and out = SwiGLU(x) (torch's silu, fp64)."""
    L = _layer(4, T=9, d=6, N=1, Z=0, I=10)
    out, r = _fwd(ref, L, 1, 0, 1)
    assert np.all(r.gate == 1.0)
    x = torch.from_numpy(L["x"])
    Wg, Wu, Wd = (torch.from_numpy(L[k][0]) for k in ("W_gate", "W_up", "W_down"))
    want = (F.silu(x @ Wg.T) * (x @ Wu.T)) @ Wd.T
    np.testing.assert_allclose(out, want.numpy(), rtol=1e-12, atol=1e-13)


def pin_all_zero_picks_closed_form(ref):
    """Zero experts boosted past every FFN expert: out = (sum of picked p) * x.

    With the same bias on all zero experts, the picks are the K zero experts
    of largest softmax probability (computed here with torch.softmax).
    """
    N, Z, K = 4, 5, 3
    L = _layer(5, T=20, d=7, N=N, Z=Z, I=8)
    L["b"] = np.concatenate([np.zeros(N), np.full(Z, 10.0)])
    out, r = _fwd(ref, L, N, Z, K)
    assert np.all(r.idx >= N)
    p = torch.softmax(torch.from_numpy(L["x"] @ L["W_r"].T), dim=1).numpy()
    top = np.sort(p[:, N:], axis=1)[:, ::-1][:, :K].sum(axis=1)
    np.testing.assert_allclose(out, top[:, None] * L["x"], rtol=1e-12, atol=1e-14)


def pin_dense_limit(ref):
    """K = E: every expert is picked, gates sum to 1, out = sum_i p_i E_i(x)."""
    N, Z = 3, 2
    E = N + Z
    L = _layer(6, T=8, d=5, N=N, Z=Z, I=6)
    out, r = _fwd(ref, L, N, Z, E)
    np.testing.assert_allclose(r.gate.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    x = torch.from_numpy(L["x"])
    p = torch.softmax(x @ torch.from_numpy(L["W_r"]).T, dim=1)
    want = p[:, N:].sum(dim=1, keepdim=True) * x
    for e in range(N):
        Wg, Wu, Wd = (torch.from_numpy(L[k][e]) for k in ("W_gate", "W_up", "W_down"))
        want = want + p[:, e:e + 1] * ((F.silu(x @ Wg.T) * (x @ Wu.T)) @ Wd.T)
    np.testing.assert_allclose(out, want.numpy(), rtol=1e-12, atol=1e-13)


def pin_textbook_moe(ref):
    """Z=0, b=0: a textbook softmax top-K MoE written with torch.topk."""
    N, K = 6, 2
    L = _layer(7, T=30, d=8, N=N, Z=0, I=12)
    L["b"] = np.zeros(N)
    out, r = _fwd(ref, L, N, 0, K)
    x = torch.from_numpy(L["x"])
    p = torch.softmax(x @ torch.from_numpy(L["W_r"]).T, dim=1)
    vals, inds = torch.topk(p, K, dim=1)
    want = torch.zeros_like(x)
    for t in range(x.shape[0]):
        for v, e in zip(vals[t], inds[t]):
            Wg, Wu, Wd = (torch.from_numpy(L[k][int(e)]) for k in ("W_gate", "W_up", "W_down"))
            want[t] += v * ((F.silu(x[t] @ Wg.T) * (x[t] @ Wu.T)) @ Wd.T)
    assert (np.sort(r.idx, 1) == np.sort(inds.numpy(), 1)).all()
    np.testing.assert_allclose(out, want.numpy(), rtol=1e-12, atol=1e-13)


def pin_logit_offset(ref):
    """An offset on the logits equals one extra input feature fixed at 1."""
    N, Z, K = 5, 3, 3
    L = _layer(8, T=25, d=6, N=N, Z=Z, I=4)
    off = _rng(9).uniform(-2, 2, N + Z)
    r1 = ref.route(L["x"], L["W_r"], L["b"], N, K, logit_offset=off)
    x2 = np.concatenate([L["x"], np.ones((25, 1))], axis=1)
    W2 = np.concatenate([L["W_r"], off[:, None]], axis=1)
    r2 = ref.route(x2, W2, L["b"], N, K)
    assert (r1.idx == r2.idx).all()
    np.testing.assert_allclose(r1.gate, r2.gate, rtol=1e-12, atol=0)


def pin_invariants(ref):
    """Counting, range and symmetry facts that hold for any input."""
    N, Z, K, d, I, T = 6, 4, 3, 5, 7, 64
    L = _layer(10, T=T, d=d, N=N, Z=Z, I=I, b_scale=0.3)
    out, r = _fwd(ref, L, N, Z, K)
    E = N + Z
    # K distinct picks per token
    assert all(len(set(row)) == K for row in r.idx.tolist())
    # histogram: all picks counted; FFN share is T*K minus zero picks
    cnt = ref.expert_load(r.idx, E)
    assert cnt.sum() == T * K
    assert cnt[:N].sum() == T * K - int((r.idx >= N).sum())
    # gates are softmax probabilities at the picks
    assert np.all(r.gate > 0) and np.all(r.gate <= 1)
    assert np.all(r.gate.sum(axis=1) <= 1 + 1e-12)
    np.testing.assert_allclose(r.p.sum(axis=1), 1.0, rtol=0, atol=1e-13)
    # permuting FFN experts (weights, bias, router rows together) permutes indices only
    perm = _rng(11).permutation(N)
    full = np.concatenate([perm, np.arange(N, E)])
    L2 = dict(L)
    L2["W_r"], L2["b"] = L["W_r"][full], L["b"][full]
    L2["W_gate"], L2["W_up"], L2["W_down"] = L["W_gate"][perm], L["W_up"][perm], L["W_down"][perm]
    out2, r2 = _fwd(ref, L2, N, Z, K)
    np.testing.assert_allclose(out2, out, rtol=1e-12, atol=1e-13)
    assert (np.sort(full[r2.idx], 1) == np.sort(r.idx, 1)).all()
    # permuting tokens permutes rows
    tp = _rng(12).permutation(T)
    L3 = dict(L)
    L3["x"] = L["x"][tp]
    out3, _ = _fwd(ref, L3, N, Z, K)
    np.testing.assert_allclose(out3, out[tp], rtol=1e-12, atol=1e-13)
    # raising the zero experts' bias never lowers a token's zero-pick count
    prev = (r.idx >= N).sum(axis=1)
    for dlt in (0.05, 0.1, 0.2, 0.5):
        L4 = dict(L)
        L4["b"] = L["b"] + np.concatenate([np.zeros(N), np.full(Z, dlt)])
        r4 = ref.route(L4["x"], L4["W_r"], L4["b"], N, K)
        now = (r4.idx >= N).sum(axis=1)
        assert np.all(now >= prev)
        prev = now
    # the gates do not move when only the bias moves (selection-only bias)
    r5 = ref.route(L["x"], L["W_r"], L["b"] * 0.0, N, K)
    np.testing.assert_allclose(r5.p, r.p, rtol=0, atol=0)


def pin_zero_expert_is_identity(ref):
    """A token whose picks are one FFN expert plus zero experts gets
    out = g_ffn E(x) + (sum of zero gates) x; checked against torch."""
    N, Z, K = 2, 3, 3
    L = _layer(13, T=10, d=4, N=N, Z=Z, I=5)
    # expert 0 always wins, expert 1 never; zero experts fill the other picks
    L["b"] = np.array([5.0, -5.0, 1.0, 1.0, 1.0])
    out, r = _fwd(ref, L, N, Z, K)
    x = torch.from_numpy(L["x"])
    p = torch.softmax(x @ torch.from_numpy(L["W_r"]).T, dim=1)
    zero_top = torch.topk(p[:, N:], K - 1, dim=1).values.sum(dim=1, keepdim=True)
    Wg, Wu, Wd = (torch.from_numpy(L[k][0]) for k in ("W_gate", "W_up", "W_down"))
    want = zero_top * x + p[:, :1] * ((F.silu(x @ Wg.T) * (x @ Wu.T)) @ Wd.T)
    np.testing.assert_allclose(out, want.numpy(), rtol=1e-12, atol=1e-13)


def pin_zero_pick_fraction(ref):
    """Share of picks on zero experts, counted by hand on small index arrays.

    Experts N..E-1 are the zero experts (reading R5), so index N counts as a
    zero pick and index N-1 does not.
    """
    N = 3
    cases = [
        ([[0, 3], [3, 4], [2, 1]], 3 / 6),    # 3 (== N) and 4 are zero experts
        ([[2, 1, 0]], 0.0),                   # 2 (== N - 1) is the last FFN expert
        ([[5, 4, 3]], 1.0),
        ([[3], [2], [3], [2]], 2 / 4),
        ([[4, 0, 1, 2], [0, 1, 2, 3]], 2 / 8),
    ]
    for idx, want in cases:
        got = ref.zero_pick_fraction(np.array(idx), N)
        assert got == want, (idx, got, want)
    # a routing whose every pick is a zero expert, and one with no zero experts
    L = _layer(14, T=12, d=4, N=N, Z=4, I=3)
    r = ref.route(L["x"], L["W_r"], np.concatenate([np.zeros(N), np.full(4, 10.0)]), N, 2)
    assert ref.zero_pick_fraction(r.idx, N) == 1.0
    r = ref.route(L["x"], L["W_r"], np.concatenate([np.full(N, 10.0), np.zeros(4)]), N, 2)
    assert ref.zero_pick_fraction(r.idx, N) == 0.0


def pin_zero_share_ties(ref):
    """The calibration's zero-expert share on score tables solved by hand.

    N = 2 FFN experts, Z = 2 zero experts, scores in sixteenths (exact in
    binary).  Row 0 scores every expert alike, row 1 is [6, 1, 5, 4]; the
    shift delta is added to the zero experts (2 and 3).  Equal scores go to
    the lower index (reading R6), so an FFN expert beats a zero expert it
    ties with.  For example K = 1, delta = 1/16: row 0 picks expert 2 (zero),
    row 1 has s = [6, 1, 6, 5] and picks expert 0 (tie, lower index): 1/2.
    """
    from oracle import calibrate_bias_shift as cal
    p = np.array([[4.0, 4.0, 4.0, 4.0], [6.0, 1.0, 5.0, 4.0]]) / 16.0
    b0 = np.zeros(4)
    cases = [
        (1, 0.0, 0 / 2),     # row 0: four-way tie -> expert 0; row 1 -> expert 0
        (1, 1.0, 1 / 2),     # row 0 -> 2; row 1: tie 0 vs 2 -> 0
        (2, 1.0, 3 / 4),     # row 0 -> {2, 3}; row 1 -> {0, 2}
        (2, 2.0, 3 / 4),     # row 1: s = [6, 1, 7, 6] -> 2, then tie 0 vs 3 -> 0
        (3, 2.0, 4 / 6),     # row 1 -> {2, 0, 3}; row 0 -> {2, 3, 0}
        (2, -1.0, 1 / 4),    # row 0: s = [4, 4, 3, 3] -> {0, 1}; row 1 -> {0, 2}
        (4, -3.0, 2 / 4),    # K = E: every expert is picked whatever the shift
    ]
    for K, shift16, want in cases:
        got = cal.zero_share(p.copy(), b0, 2, K, shift16 / 16.0)
        assert got == want, (K, shift16, got, want)


ALL_PINS = [
    pin_worked_examples,
    pin_topk_brute_force,
    pin_topk_ties_lower_index,
    pin_scalar_loops,
    pin_single_expert_is_swiglu,
    pin_all_zero_picks_closed_form,
    pin_dense_limit,
    pin_textbook_moe,
    pin_logit_offset,
    pin_invariants,
    pin_zero_expert_is_identity,
    pin_zero_pick_fraction,
    pin_zero_share_ties,
]
