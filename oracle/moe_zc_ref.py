"""Plain fp64 definition of the MoE layer with zero-computation experts.

TEST INFRASTRUCTURE ONLY (see the package docstring): the CUDA library never
imports this file.

Source: the LongCat-Flash write-up "Meituan's large model goes viral for its
speed" (itouyu.top), section "Zero-computation experts".  It says that the
expert pool holds N standard FFN experts plus Z zero-computation experts that
return their input unchanged; that R is a softmax router, b_i the bias of
expert i and K the number of experts each token picks; that the number of FFN
experts a token uses therefore varies; and that the bias adjusts the routing
scores from recent expert usage while staying out of the training loss.  The
formula that followed "can be formalised as follows" is missing from every
copy of the page, so the layer is rebuilt from that glossary.

Readings taken where the page is silent (each one is also a test):
  R1  the softmax runs over all E = N + Z experts (the zero experts are part
      of the pool the router scores);
  R2  the bias is added after the softmax, to the routing score s = p + b;
  R3  the bias changes only which experts are picked: gate g_i = p_i, taken
      from the one unbiased softmax, with no renormalisation over the picks;
  R4  an FFN expert is SwiGLU without biases:
      E_i(x) = W_down,i (SiLU(W_gate,i x) * (W_up,i x)), SiLU(z) = z/(1+e^-z);
  R5  experts 0..N-1 are FFN experts, N..E-1 are zero experts;
  R6  the top-K takes the K largest s; equal scores go to the lower index;
  R7  the expert-load histogram counts picks of all E experts (the bias
      controller needs zero-expert usage too);
  R8  an optional per-expert logit offset is added to the logits before the
      softmax (used only to skew expert load in a synthetic workload).

Everything is computed in float64 from the exact bf16 / fp32 input values.
Library routines used as steps: numpy matmul, exp, argsort (stable).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Optional, Sequence

import numpy as np


def _f64(a) -> np.ndarray:
    """Widen an array-like (numpy or CPU torch tensor) to float64 numpy."""
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").double().numpy()
    return np.asarray(a, dtype=np.float64)


def router_logits(x, W_r, logit_offset=None) -> np.ndarray:
    """l_t = x_t W_r^T (+ offset): one score per expert of the pool (R1, R8).

    Section "Zero-computation experts": R scores every expert of the pool.
    x [T, d], W_r [E, d] -> l [T, E].
    """
    l = _f64(x) @ _f64(W_r).T
    if logit_offset is not None:
        l = l + _f64(logit_offset)[None, :]
    return l


def softmax(l: np.ndarray) -> np.ndarray:
    """p_t = softmax(l_t) over all E experts (R1), as exp(l-max)/sum exp(l-max)."""
    m = l.max(axis=1, keepdims=True)
    e = np.exp(l - m)
    return e / e.sum(axis=1, keepdims=True)


def select_topk(s: np.ndarray, K: int):
    """Indices of the K largest scores per row, largest first (R6).

    Equal scores go to the lower index: a stable sort of -s keeps equal keys
    in index order.  Also returns gap = s(K-th) - s((K+1)-th), +inf when K = E;
    the gap measures how close a token is to a tie at the selection boundary.
    """
    T, E = s.shape
    order = np.argsort(-s, axis=1, kind="stable")
    idx = order[:, :K]
    if K < E:
        kth = np.take_along_axis(s, order[:, K - 1:K], axis=1)[:, 0]
        nxt = np.take_along_axis(s, order[:, K:K + 1], axis=1)[:, 0]
        gap = kth - nxt
    else:
        gap = np.full(T, np.inf)
    return idx, gap


@dataclass
class Routing:
    idx: np.ndarray     # [T, K] int64, largest biased score first
    gate: np.ndarray    # [T, K] float64, g = p at the picks
    gap: np.ndarray     # [T] float64, s(K) - s(K+1)
    p: np.ndarray       # [T, E] float64, the unbiased softmax
    N: int

    @property
    def zsum(self) -> np.ndarray:
        """Sum of the gates a token puts on zero experts (idx >= N)."""
        return np.where(self.idx >= self.N, self.gate, 0.0).sum(axis=1)


def route(x, W_r, b, N: int, K: int, logit_offset=None) -> Routing:
    """Router of section "Zero-computation experts": softmax, +b, top-K.

    s = p + b selects (R2); the gates are the unbiased p at the picks (R3).
    """
    p = softmax(router_logits(x, W_r, logit_offset))
    s = p + _f64(b)[None, :]
    idx, gap = select_topk(s, K)
    gate = np.take_along_axis(p, idx, axis=1)
    return Routing(idx=idx, gate=gate, gap=gap, p=p, N=N)


def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def swiglu_expert(xs, Wg, Wu, Wd) -> np.ndarray:
    """E_i(x) = W_down (SiLU(W_gate x) * (W_up x)) for each row of xs (R4).

    xs [n, d], Wg [I, d], Wu [I, d], Wd [d, I] -> [n, d].
    """
    xs = _f64(xs)
    a = xs @ _f64(Wg).T
    u = xs @ _f64(Wu).T
    return (silu(a) * u) @ _f64(Wd).T


def forward_rows(x, r: Routing, expert: Callable[[int], Sequence[np.ndarray]]) -> np.ndarray:
    """out_t = sum over picks of g_i E_i(x_t), for the rows of x routed by r.

    A zero expert returns its input, so its term is g_i x_t (section
    "Zero-computation experts"); an FFN expert's term is g_i E_i(x_t) (R4).
    ``expert(e)`` returns (W_gate[e], W_up[e], W_down[e]); it is called once
    per FFN expert that some row picks, so callers can fetch weights lazily.
    """
    xs = _f64(x)
    out = r.zsum[:, None] * xs
    N = r.N
    for e in np.unique(r.idx[r.idx < N]):
        rows, ks = np.nonzero(r.idx == e)
        Wg, Wu, Wd = expert(int(e))
        out[rows] += r.gate[rows, ks][:, None] * swiglu_expert(xs[rows], Wg, Wu, Wd)
    return out


def forward(x, W_r, b, W_gate, W_up, W_down, N: int, Z: int, K: int,
            logit_offset=None):
    """The whole layer: (out [T, d] float64, Routing).

    W_gate [N, I, d], W_up [N, I, d], W_down [N, d, I]; b [N+Z].
    """
    assert _f64(W_r).shape[0] == N + Z
    r = route(x, W_r, b, N, K, logit_offset)
    out = forward_rows(x, r, lambda e: (W_gate[e], W_up[e], W_down[e]))
    return out, r


def expert_load(idx: np.ndarray, E: int) -> np.ndarray:
    """cnt_i = number of tokens that pick expert i, for all E experts (R7).

    Section "Zero-computation experts": the bias follows recent expert usage.
    """
    return np.bincount(np.asarray(idx).ravel(), minlength=E).astype(np.int64)


def zero_pick_fraction(idx: np.ndarray, N: int) -> float:
    """Share of all T*K picks that land on zero experts (indices N..E-1, R5).

    Section "Zero-computation experts": a token's picks split between FFN
    experts and zero experts, so the number of FFN experts it runs varies;
    this is the share of the pool's picks the zero experts take.
    """
    idx = np.asarray(idx)
    return float((idx >= N).sum()) / max(idx.size, 1)
