"""fp64 definition of the PID bias controller (test infrastructure only).

LongCat-Flash write-up "Meituan's large model goes viral for its speed",
section "Zero-computation experts": expert biases follow recent expert usage
through a PID controller.  The page gives no gains, set-point or window; the
reading taken (the same as the library's controller states):

  set-point  L*_i = (1 - rho) T K / N for FFN experts, rho T K / Z for zero experts
  error      e_i = (L*_i - L_i) / (T K / E)
  law        b_i = base_i + clip(kp e_i + ki sum_s e_i(s) + kd (e_i - e_i,prev))

with conditional integration (the textbook remedy for integral windup of a
clipped PID): a step whose unclipped output would lie beyond the clip on the
side its error pushes towards leaves the integral as it was, so that after a
long saturated stretch the bias leaves the clip as soon as the error turns.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


@dataclass
class PidState:
    base: np.ndarray                 # bias when the controller started
    integral: np.ndarray = None      # running sum of the error
    prev: np.ndarray = None          # last step's error

    def __post_init__(self):
        self.base = np.asarray(self.base, dtype=np.float64).copy()
        if self.integral is None:
            self.integral = np.zeros_like(self.base)
        if self.prev is None:
            self.prev = np.zeros_like(self.base)


def target_load(N: int, Z: int, tokens: int, K: int, rho: float) -> np.ndarray:
    """Set-point: zero experts share rho of the picks, FFN experts the rest, evenly."""
    picks = float(tokens) * K
    t = np.empty(N + Z)
    if N:
        t[:N] = (1.0 - rho) * picks / N
    if Z:
        t[N:] = rho * picks / Z
    return t


def step(state: PidState, counts, N: int, Z: int, tokens: int, K: int, rho: float,
         kp: float, ki: float, kd: float, max_shift: float = 0.0) -> np.ndarray:
    """One controller step: update the state, return the new biases."""
    counts = np.asarray(counts, dtype=np.float64)
    E = N + Z
    e = (target_load(N, Z, tokens, K, rho) - counts) / (float(tokens) * K / E)
    integral = state.integral + e
    shift = kp * e + ki * integral + kd * (e - state.prev)
    if max_shift > 0:
        # saturated, and the error pushes further out: do not integrate
        wind = (np.abs(shift) > max_shift) & (np.sign(shift) == np.sign(e))
        integral = np.where(wind, state.integral, integral)
        shift = kp * e + ki * integral + kd * (e - state.prev)
        shift = np.clip(shift, -max_shift, max_shift)
    state.integral = integral
    state.prev = e
    return state.base + shift
