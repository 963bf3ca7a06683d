"""FP8 (E4M3) block quantisation, and the MoE layer with FP8 gate/up experts,
in plain fp64.

TEST INFRASTRUCTURE ONLY (see the package docstring): no CUDA code imports
this file.  It defines what a future FP8 expert path must compute; the CUDA
library has no FP8 path yet.

Source: the LongCat-Flash write-up "Meituan's large model goes viral for its
speed" (itouyu.top), section "System-level optimisation", its paragraph on
quantisation: the model uses the fine-grained block quantisation of
DeepSeek-V3, and a layer-wise mixed precision that keeps in higher precision
the linear layers whose input activations reach extreme magnitudes (the down
projection is the example given) and the expert layers with a large block
FP8 error.  The page gives no format, block shape or scale rule, so these
readings are taken (each one is a test):
  Q1  elements are E4M3: sign, 4 exponent bits with bias 7, 3 mantissa bits,
      no infinities, one NaN code per sign (exponent and mantissa all ones);
      exponent field 0 holds the subnormals m/8 * 2^-6; the largest finite
      magnitude is 448;
  Q2  a weight matrix [rows, cols] is cut into 128 x 128 blocks, each with
      one fp32 scale;
  Q3  activations are cut into 1 x 128 tiles (one token, 128 consecutive
      features), each with one fp32 scale;
  Q4  a block's scale is amax / 448 (amax = its largest magnitude); an
      all-zero block, or one holding a NaN or an infinity, gets scale 1;
  Q5  encoding rounds to the nearest E4M3 value, ties to the even code, and
      saturates at +-448;
  Q6  the scale and the scaled value w / scale are formed in fp32 (IEEE
      round to nearest), the precision in which a device encodes them, so
      that both sides take the same decision on every code;
  Q7  mixed precision: the gate and up projections run in FP8 (weights and
      their input tokens quantised), the down projection stays bf16.
The dequantised value of a code is decode(code) * scale, exactly, in fp64;
the layer is then the fp64 definition of moe_zc_ref on dequantised operands.

A second reading, for the tensor cores' block-scaled FP8 form, replaces Q2-Q4
(the ``mx`` functions below):
  M1  weights and activations alike are cut into 1 x 32 blocks along the
      contraction dimension (one weight row or one token, 32 consecutive
      features), each with one power-of-two scale (an 8-bit exponent);
  M2  the scale is the smallest power of two with amax / scale <= 448, so no
      element saturates; an all-zero or non-finite block gets scale 1.
Q1, Q5-Q7 hold for it unchanged (dividing by a power of two is exact).
"""
from __future__ import annotations

from typing import Callable, Sequence, Tuple

import numpy as np

from oracle import moe_zc_ref as ref

E4M3_MAX = 448.0
WEIGHT_BLOCK = (128, 128)   # Q2
ACT_TILE = (1, 128)         # Q3
MX_BLOCK = (1, 32)          # M1


def e4m3_value(code: int) -> float:
    """The value of one E4M3 code (Q1), from its bit fields."""
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)
# non-negative finite magnitudes in code order 0x00..0x7E (increasing)
_POS = _TABLE[:0x7F]


def e4m3_decode(codes) -> np.ndarray:
    """Values (float64) of an array of uint8 codes."""
    return _TABLE[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(v) -> np.ndarray:
    """uint8 codes of float32 values: nearest E4M3 value, ties to the even
    code, magnitudes beyond 448 saturated to 448 (Q5).  NaN maps to 0x7F."""
    v = np.asarray(v, dtype=np.float32)
    a = np.abs(v).astype(np.float64)
    hi = np.clip(np.searchsorted(_POS, a, side="left"), 0, len(_POS) - 1)
    lo = np.clip(hi - 1, 0, len(_POS) - 1)
    d_lo = np.abs(a - _POS[lo])
    d_hi = np.abs(_POS[hi] - a)
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    code = np.where(a >= E4M3_MAX, np.uint8(0x7E), code)
    code = np.where(np.signbit(v), code | np.uint8(0x80), code).astype(np.uint8)
    return np.where(np.isnan(v), np.uint8(0x7F), code).astype(np.uint8)


def quantize_blocks(W, block: Tuple[int, int]) -> Tuple[np.ndarray, np.ndarray]:
    """(codes uint8 [R, C], scales float32 [ceil(R/br), ceil(C/bc)]) of a 2-D
    array cut into br x bc blocks (Q4-Q6).  Ragged edge blocks are smaller."""
    W = np.asarray(W, dtype=np.float32)
    R, C = W.shape
    br, bc = block
    nr, nc = -(-R // br), -(-C // bc)
    scales = np.ones((nr, nc), dtype=np.float32)
    codes = np.zeros((R, C), dtype=np.uint8)
    for i in range(nr):
        for j in range(nc):
            blk = W[i * br:(i + 1) * br, j * bc:(j + 1) * bc]
            amax = np.float32(np.max(np.abs(blk))) if blk.size else np.float32(0)
            ok = amax > 0 and np.isfinite(amax)     # NaN or infinity: scale 1
            s = np.float32(amax / np.float32(E4M3_MAX)) if ok else np.float32(1.0)
            scales[i, j] = s
            codes[i * br:(i + 1) * br, j * bc:(j + 1) * bc] = e4m3_encode(blk / s)
    return codes, scales


def dequantize_blocks(codes, scales, block: Tuple[int, int]) -> np.ndarray:
    """decode(code) * scale of every element, in fp64."""
    codes = np.asarray(codes, dtype=np.uint8)
    br, bc = block
    s = np.repeat(np.repeat(np.asarray(scales, dtype=np.float64), br, axis=0), bc, axis=1)
    return e4m3_decode(codes) * s[: codes.shape[0], : codes.shape[1]]


def quantize_mx(W) -> Tuple[np.ndarray, np.ndarray]:
    """(codes uint8 [R, C], scales float32 [R, ceil(C/32)]) under M1-M2: each
    1 x 32 block's scale is 2^ceil(log2(amax / 448))."""
    W = np.asarray(W, dtype=np.float32)
    R, C = W.shape
    nb = -(-C // MX_BLOCK[1])
    scales = np.ones((R, nb), dtype=np.float32)
    codes = np.zeros((R, C), dtype=np.uint8)
    for j in range(nb):
        blk = W[:, j * MX_BLOCK[1]:(j + 1) * MX_BLOCK[1]]
        amax = np.max(np.abs(blk), axis=1).astype(np.float64)
        e = np.zeros(R)
        nz = (amax > 0) & np.isfinite(amax)          # NaN or infinity: scale 1
        amax = np.where(nz, amax, 0.0)
        e[nz] = np.ceil(np.log2(amax[nz] / E4M3_MAX))
        # guard the log2 rounding both ways: the smallest power of two with
        # amax / s <= 448 (divisions by powers of two are exact)
        s = np.ldexp(1.0, e.astype(int))
        higher = nz & (amax / s > E4M3_MAX)
        s[higher] *= 2
        lower = nz & (amax / (s / 2) <= E4M3_MAX)
        s[lower] /= 2
        s[~nz] = 1.0
        scales[:, j] = s.astype(np.float32)
        codes[:, j * MX_BLOCK[1]:(j + 1) * MX_BLOCK[1]] = e4m3_encode(blk / s[:, None].astype(np.float32))
    return codes, scales


def fp8_swiglu_expert_mx(xs, Wg_q, Wu_q, Wd) -> np.ndarray:
    """E(x) with FP8 gate/up under the block-scaled reading (M1-M2): tokens
    and weights in 1 x 32 blocks along d; the down projection unquantised."""
    cx, sx = quantize_mx(xs)
    Xd = dequantize_blocks(cx, sx, MX_BLOCK)
    Wg = dequantize_blocks(*Wg_q, MX_BLOCK)
    Wu = dequantize_blocks(*Wu_q, MX_BLOCK)
    H = ref.silu(Xd @ Wg.T) * (Xd @ Wu.T)
    return H @ ref._f64(Wd).T


def quantize_weight(W) -> Tuple[np.ndarray, np.ndarray]:
    """One expert matrix in 128 x 128 blocks (Q2)."""
    return quantize_blocks(W, WEIGHT_BLOCK)


def quantize_activations(X) -> Tuple[np.ndarray, np.ndarray]:
    """Token rows in 1 x 128 tiles (Q3)."""
    return quantize_blocks(X, ACT_TILE)


def fp8_swiglu_expert(xs, Wg_q, Wu_q, Wd) -> np.ndarray:
    """E(x) with FP8 gate/up (Q7): the token rows xs are quantised in 1 x 128
    tiles, the weights come quantised as (codes, scales) pairs; the down
    projection takes H and W_down unquantised."""
    cx, sx = quantize_activations(xs)
    Xd = dequantize_blocks(cx, sx, ACT_TILE)
    Wg = dequantize_blocks(*Wg_q, WEIGHT_BLOCK)
    Wu = dequantize_blocks(*Wu_q, WEIGHT_BLOCK)
    H = ref.silu(Xd @ Wg.T) * (Xd @ Wu.T)
    return H @ ref._f64(Wd).T


def forward_rows_fp8(x, r: ref.Routing, expert: Callable[[int], Sequence],
                     mx: bool = False) -> np.ndarray:
    """out_t for the rows of x routed by r (routing as in moe_zc_ref: the
    router stays bf16/fp32), FFN terms from fp8_swiglu_expert (mx: from
    fp8_swiglu_expert_mx).  ``expert(e)`` returns ((codes, scales) of
    W_gate[e], (codes, scales) of W_up[e], W_down[e]), quantised with
    quantize_weight (mx: quantize_mx)."""
    xs = ref._f64(x)
    xq = xs.astype(np.float32)      # exact: x holds bf16 values
    out = r.zsum[:, None] * xs
    term = fp8_swiglu_expert_mx if mx else fp8_swiglu_expert
    for e in np.unique(r.idx[r.idx < r.N]):
        rows, ks = np.nonzero(r.idx == e)
        Wg_q, Wu_q, Wd = expert(int(e))
        out[rows] += r.gate[rows, ks][:, None] * term(xq[rows], Wg_q, Wu_q, Wd)
    return out
