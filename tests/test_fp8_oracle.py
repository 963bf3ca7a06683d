"""Pins of the FP8 oracle (oracle/fp8_ref.py): the E4M3 code table and
encoder against torch's float8_e4m3fn type and brute force, the block and
tile quantisation against closed forms and invariances, and the FP8 layer
against the bf16 layer where quantisation is exact."""
import numpy as np
import pytest
import torch

from oracle import fp8_ref as f8
from oracle import moe_zc_ref as ref


def _torch_codes(v):
    return torch.from_numpy(np.asarray(v, dtype=np.float32)).to(torch.float8_e4m3fn) \
        .view(torch.uint8).numpy()


def test_decode_table_matches_torch_float8():
    codes = np.arange(256, dtype=np.uint8)
    tv = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    mine = f8.e4m3_decode(codes)
    assert np.array_equal(np.isnan(tv), np.isnan(mine))
    assert np.array_equal(tv[~np.isnan(tv)], mine[~np.isnan(mine)])
    # closed-form landmarks: largest finite, smallest normal and subnormal
    assert mine[0x7E] == 448.0 and mine[0x08] == 2.0 ** -6 and mine[0x01] == 2.0 ** -9
    assert np.isnan(mine[0x7F]) and np.isnan(mine[0xFF]) and mine[0x80] == 0.0


def test_encode_matches_torch_in_range():
    g = np.random.default_rng(0)
    v = np.concatenate([g.standard_normal(50000).astype(np.float32) * s
                        for s in (1e-3, 0.05, 1.0, 30.0, 200.0)])
    v = v[np.abs(v) < 448]
    assert np.array_equal(f8.e4m3_encode(v), _torch_codes(v))
    # every midpoint between neighbouring values: ties go to the even code
    pos = f8.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mids = (pos[:-1] + pos[1:]) / 2
    assert np.array_equal(mids.astype(np.float32).astype(np.float64), mids)
    c = f8.e4m3_encode(mids)
    assert np.array_equal(c, _torch_codes(mids))
    assert np.all(c % 2 == 0)


def test_encode_saturates_and_keeps_sign():
    c = f8.e4m3_encode(np.array([449.0, 464.0, 500.0, 1e6, -1e6, -0.0, np.nan], np.float32))
    assert list(c) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x80, 0x7F]


def test_encode_is_a_nearest_value():
    g = np.random.default_rng(1)
    v = (g.standard_normal(4000) * 10.0 ** g.uniform(-3, 2.5, 4000)).astype(np.float32)
    v = v[np.abs(v) < 448]
    got = f8.e4m3_decode(f8.e4m3_encode(v))
    table = f8.e4m3_decode(np.arange(256, dtype=np.uint8))
    table = table[~np.isnan(table)]
    best = np.min(np.abs(table[None, :] - v.astype(np.float64)[:, None]), axis=1)
    assert np.array_equal(np.abs(got - v), best)


def _gauss(shape, seed, scale=1.0):
    g = np.random.default_rng(seed)
    return (g.standard_normal(shape) * scale).astype(np.float32)


def test_block_maximum_maps_to_448_and_error_bound():
    W = _gauss((256, 384), 2, 0.02)
    codes, scales = f8.quantize_weight(W)
    assert scales.shape == (2, 3) and scales.dtype == np.float32
    deq = f8.dequantize_blocks(codes, scales, f8.WEIGHT_BLOCK)
    for i in range(2):
        for j in range(3):
            blk = W[128 * i:128 * (i + 1), 128 * j:128 * (j + 1)].astype(np.float64)
            cb = codes[128 * i:128 * (i + 1), 128 * j:128 * (j + 1)]
            amax = np.abs(blk).max()
            assert scales[i, j] == np.float32(np.float32(amax) / np.float32(448))
            k = np.unravel_index(np.argmax(np.abs(blk)), blk.shape)
            assert cb[k] & 0x7F == 0x7E
            d = deq[128 * i:128 * (i + 1), 128 * j:128 * (j + 1)]
            s = float(scales[i, j])
            normal = np.abs(blk) >= 2.0 ** -6 * s
            # 3 mantissa bits: half a unit in the last place, relative 2^-4
            assert np.all(np.abs(d - blk)[normal] <= 2.0 ** -4 * np.abs(blk)[normal] * (1 + 1e-6))
            # subnormal spacing 2^-9: half of it, times the scale
            assert np.all(np.abs(d - blk)[~normal] <= 2.0 ** -10 * s * (1 + 1e-6))


def test_dequantised_blocks_keep_their_own_scale():
    """A square grid of blocks of very different magnitudes: each block comes
    back within E4M3 rounding of itself."""
    W = _gauss((256, 256), 9)
    for i in range(2):
        for j in range(2):
            W[128 * i:128 * (i + 1), 128 * j:128 * (j + 1)] *= np.float32(4.0 ** (2 * i + j))
    codes, scales = f8.quantize_weight(W)
    deq = f8.dequantize_blocks(codes, scales, f8.WEIGHT_BLOCK)
    W64 = W.astype(np.float64)
    normal = np.abs(W64) >= 2.0 ** -6 * np.repeat(np.repeat(scales, 128, 0), 128, 1)
    assert np.all(np.abs(deq - W64)[normal] <= 2.0 ** -4 * np.abs(W64)[normal] * (1 + 1e-6))


def test_power_of_two_rescaling_keeps_codes():
    W = _gauss((128, 256), 3)
    c1, s1 = f8.quantize_weight(W)
    c2, s2 = f8.quantize_weight(W * np.float32(8.0))
    assert np.array_equal(c1, c2) and np.array_equal(s2, s1 * np.float32(8.0))


def test_blocks_and_tiles_are_independent():
    W = _gauss((200, 300), 4)                       # ragged edge blocks
    c1, s1 = f8.quantize_weight(W)
    assert s1.shape == (2, 3)
    W2 = W.copy()
    W2[5, 7] = 50.0                                 # only block (0, 0) changes
    c2, s2 = f8.quantize_weight(W2)
    keep = np.ones_like(s1, dtype=bool)
    keep[0, 0] = False
    assert np.array_equal(s1[keep], s2[keep]) and s1[0, 0] != s2[0, 0]
    assert np.array_equal(c1[128:], c2[128:]) and np.array_equal(c1[:128, 128:], c2[:128, 128:])
    # activations: 1 x 128 tiles, one token each
    X = _gauss((6, 256), 5)
    cx, sx = f8.quantize_activations(X)
    assert sx.shape == (6, 2)
    X2 = X.copy()
    X2[3] *= np.float32(4.0)
    cx2, sx2 = f8.quantize_activations(X2)
    assert np.array_equal(cx, cx2)
    assert np.array_equal(np.delete(sx, 3, 0), np.delete(sx2, 3, 0))
    assert np.array_equal(sx2[3], sx[3] * np.float32(4.0))


def _on_grid(shape, seed, exp, block):
    """Values v * 2^exp with v drawn from the E4M3 table, each block holding
    one +-448 * 2^exp, so that the block scale is exactly 2^exp."""
    g = np.random.default_rng(seed)
    table = f8.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    v = g.choice(table, size=shape) * g.choice([-1.0, 1.0], size=shape)
    br, bc = block
    for i in range(0, shape[0], br):
        for j in range(0, shape[1], bc):
            v[i, j] = 448.0
    return (v * 2.0 ** exp).astype(np.float32)


def test_fp8_layer_equals_bf16_layer_when_quantisation_is_exact():
    T, d, I, N, Z, K = 24, 256, 256, 4, 2, 3
    x = torch.from_numpy(_on_grid((T, d), 6, -8, f8.ACT_TILE)).to(torch.bfloat16)
    assert np.array_equal(x.float().numpy(), _on_grid((T, d), 6, -8, f8.ACT_TILE))
    Wg = [_on_grid((I, d), 10 + e, -12, f8.WEIGHT_BLOCK) for e in range(N)]
    Wu = [_on_grid((I, d), 20 + e, -12, f8.WEIGHT_BLOCK) for e in range(N)]
    Wd = [_gauss((d, I), 30 + e, 0.02) for e in range(N)]
    g = torch.Generator().manual_seed(7)
    W_r = (torch.randn(N + Z, d, generator=g) * 0.05).to(torch.bfloat16)
    b = torch.zeros(N + Z)
    r = ref.route(x, W_r, b, N, K)
    assert (r.idx < N).any()
    q = {e: (f8.quantize_weight(Wg[e]), f8.quantize_weight(Wu[e]), Wd[e]) for e in range(N)}
    for e in range(N):
        assert np.all(q[e][0][1] == np.float32(2.0 ** -12))
    out8 = f8.forward_rows_fp8(x, r, lambda e: q[e])
    out = ref.forward_rows(x, r, lambda e: (Wg[e], Wu[e], Wd[e]))
    assert np.allclose(out8, out, rtol=1e-12, atol=1e-15)


def test_fp8_layer_on_gaussian_weights_differs_by_e4m3_rounding():
    T, d, I, N, Z, K = 32, 256, 128, 4, 2, 3
    g = torch.Generator().manual_seed(8)
    x = torch.randn(T, d, generator=g).to(torch.bfloat16)
    W_r = (torch.randn(N + Z, d, generator=g) * 0.05).to(torch.bfloat16)
    Wg = [_gauss((I, d), 40 + e, 0.02) for e in range(N)]
    Wu = [_gauss((I, d), 50 + e, 0.02) for e in range(N)]
    Wd = [_gauss((d, I), 60 + e, 0.02) for e in range(N)]
    r = ref.route(x, W_r, torch.zeros(N + Z), N, K)
    q = {e: (f8.quantize_weight(Wg[e]), f8.quantize_weight(Wu[e]), Wd[e]) for e in range(N)}
    out8 = f8.forward_rows_fp8(x, r, lambda e: q[e])
    out = ref.forward_rows(x, r, lambda e: (Wg[e], Wu[e], Wd[e]))
    ffn = (r.idx < N).any(axis=1)
    zero_terms = r.zsum[:, None] * x.double().numpy()
    term8, term = (out8 - zero_terms)[ffn], (out - zero_terms)[ffn]
    rel = np.sqrt(np.mean((term8 - term) ** 2)) / np.sqrt(np.mean(term ** 2))
    # E4M3 rounds each operand by up to 2^-4 relative (rms ~2^-4/sqrt(3)
    # for uniform rounding); the FFN terms inherit a few percent
    assert 5e-3 < rel < 0.08
    # rows with zero-expert picks only are untouched
    assert np.array_equal(out8[~ffn], out[~ffn])


# --------------------------------------------------------------- mutants
# Plausible mistakes planted in the FP8 oracle; each must fail some pin above.

_PINS = [test_decode_table_matches_torch_float8, test_encode_matches_torch_in_range,
         test_encode_saturates_and_keeps_sign, test_encode_is_a_nearest_value,
         test_block_maximum_maps_to_448_and_error_bound,
         test_dequantised_blocks_keep_their_own_scale, test_power_of_two_rescaling_keeps_codes,
         test_blocks_and_tiles_are_independent,
         test_fp8_layer_equals_bf16_layer_when_quantisation_is_exact,
         test_fp8_layer_on_gaussian_weights_differs_by_e4m3_rounding]

_orig_encode = f8.e4m3_encode
_orig_swiglu = f8.fp8_swiglu_expert
_orig_quant = f8.quantize_blocks
_orig_deq = f8.dequantize_blocks


def _encode_ties_odd(v):
    c = _orig_encode(v)
    a = np.abs(np.asarray(v, np.float32)).astype(np.float64)
    pos = f8._POS
    hi = np.clip(np.searchsorted(pos, a), 0, len(pos) - 1)
    lo = np.clip(hi - 1, 0, len(pos) - 1)
    tie = (np.abs(a - pos[lo]) == np.abs(pos[hi] - a)) & (hi != lo) & (a < 448)
    return np.where(tie, c ^ np.uint8(1), c).astype(np.uint8)


def _encode_no_saturation(v):
    c = _orig_encode(v)
    return np.where(np.abs(np.asarray(v, np.float32)) > 464, c | np.uint8(0x7F), c).astype(np.uint8)


def _quant_scale_256(W, block):
    codes, scales = _orig_quant(np.asarray(W, np.float32) * np.float32(448 / 256), block)
    return codes, (scales / np.float32(448 / 256)).astype(np.float32)


def _deq_scales_transposed(codes, scales, block):
    s = np.asarray(scales)
    if s.shape[0] != s.shape[1]:
        return _orig_deq(codes, s, block)
    return _orig_deq(codes, s.T, block)


def _swiglu_down_quantised(xs, Wg_q, Wu_q, Wd):
    cd, sd = f8.quantize_weight(np.asarray(ref._f64(Wd), np.float32))
    return _orig_swiglu(xs, Wg_q, Wu_q, f8.dequantize_blocks(cd, sd, f8.WEIGHT_BLOCK))


def _subnormal_table():
    t = f8._TABLE.copy()
    for c in list(range(1, 8)) + list(range(0x81, 0x88)):
        m = c & 7
        t[c] = (-1.0 if c & 0x80 else 1.0) * (1.0 + m / 8.0) * 2.0 ** -7
    return t


MUTANTS = {
    "ties to the odd code": dict(e4m3_encode=_encode_ties_odd),
    "no saturation at 448": dict(e4m3_encode=_encode_no_saturation),
    "scale amax / 256": dict(quantize_blocks=_quant_scale_256),
    "activation tiles 128 x 1": dict(ACT_TILE=(128, 1)),
    "subnormals decoded as normals": dict(_TABLE="subnormal"),
    "block scales transposed": dict(dequantize_blocks=_deq_scales_transposed),
    "down projection quantised too": dict(fp8_swiglu_expert=_swiglu_down_quantised),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_fp8_mutant_is_caught(name, monkeypatch):
    for attr, val in MUTANTS[name].items():
        if val == "subnormal":
            t = _subnormal_table()
            monkeypatch.setattr(f8, "_TABLE", t)
            monkeypatch.setattr(f8, "_POS", t[:0x7F])
        else:
            monkeypatch.setattr(f8, attr, val)
    caught = []
    for pin in _PINS:
        try:
            pin()
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches: {name}"


# ------------------------------------------------- block-scaled reading (M1-M2)

def test_mx_scales_are_the_smallest_powers_of_two_without_saturation():
    W = _gauss((16, 200), 11, 0.02)                  # ragged last block of 8
    W[3, 64:96] = 0.0                                 # an all-zero block
    codes, scales = f8.quantize_mx(W)
    assert scales.shape == (16, 7)
    e = np.log2(scales.astype(np.float64))
    assert np.array_equal(e, np.round(e))
    assert scales[3, 2] == 1.0 and np.all(codes[3, 64:96] & 0x7F == 0)
    for j in range(7):
        amax = np.abs(W[:, 32 * j:32 * (j + 1)]).max(axis=1).astype(np.float64)
        nz = amax > 0
        s = scales[nz, j].astype(np.float64)
        assert np.all(amax[nz] / s <= 448.0) and np.all(amax[nz] / (s / 2) > 448.0)
    deq = f8.dequantize_blocks(codes, scales, f8.MX_BLOCK)
    s_el = np.repeat(scales.astype(np.float64), 32, axis=1)[:, :200]
    W64 = W.astype(np.float64)
    normal = np.abs(W64) >= 2.0 ** -6 * s_el
    assert np.all(np.abs(deq - W64)[normal] <= 2.0 ** -4 * np.abs(W64)[normal] * (1 + 1e-6))
    assert np.all(np.abs(deq - W64)[~normal] <= 2.0 ** -10 * s_el[~normal] * (1 + 1e-6))


def test_mx_blocks_run_along_the_contraction_dimension():
    X = _gauss((5, 128), 12)
    c1, s1 = f8.quantize_mx(X)
    X2 = X.copy()
    X2[2, 40] = 100.0                                 # block (row 2, features 32..63)
    c2, s2 = f8.quantize_mx(X2)
    diff = s1 != s2
    assert diff.sum() == 1 and diff[2, 1]


def test_mx_layer_equals_bf16_layer_when_quantisation_is_exact():
    T, d, I, N, Z, K = 20, 128, 128, 3, 2, 2
    xv = _on_grid((T, d), 13, -8, f8.MX_BLOCK)
    x = torch.from_numpy(xv).to(torch.bfloat16)
    assert np.array_equal(x.float().numpy(), xv)
    Wg = [_on_grid((I, d), 14 + e, -12, f8.MX_BLOCK) for e in range(N)]
    Wu = [_on_grid((I, d), 24 + e, -12, f8.MX_BLOCK) for e in range(N)]
    Wd = [_gauss((d, I), 34 + e, 0.02) for e in range(N)]
    g = torch.Generator().manual_seed(9)
    W_r = (torch.randn(N + Z, d, generator=g) * 0.05).to(torch.bfloat16)
    r = ref.route(x, W_r, torch.zeros(N + Z), N, K)
    assert (r.idx < N).any()
    q = {e: (f8.quantize_mx(Wg[e]), f8.quantize_mx(Wu[e]), Wd[e]) for e in range(N)}
    assert all(np.all(q[e][0][1] == np.float32(2.0 ** -12)) for e in range(N))
    out8 = f8.forward_rows_fp8(x, r, lambda e: q[e], mx=True)
    out = ref.forward_rows(x, r, lambda e: (Wg[e], Wu[e], Wd[e]))
    assert np.allclose(out8, out, rtol=1e-12, atol=1e-15)


def _mx_scale_floor(W):
    """Mutant: the OCP-style floor exponent, 2^(floor(log2 amax) - 8), which
    lets the largest elements saturate."""
    W = np.asarray(W, dtype=np.float32)
    codes, scales = _orig_mx(W)
    R, C = W.shape
    for j in range(scales.shape[1]):
        blk = W[:, 32 * j:32 * (j + 1)]
        amax = np.abs(blk).max(axis=1).astype(np.float64)
        s = np.where(amax > 0, np.ldexp(1.0, (np.floor(np.log2(np.maximum(amax, 1e-300))) - 8)
                                        .astype(int)), 1.0)
        scales[:, j] = s
        codes[:, 32 * j:32 * (j + 1)] = f8.e4m3_encode(blk / s[:, None].astype(np.float32))
    return codes, scales


_orig_mx = f8.quantize_mx
_MX_PINS = [test_mx_scales_are_the_smallest_powers_of_two_without_saturation,
            test_mx_blocks_run_along_the_contraction_dimension,
            test_mx_layer_equals_bf16_layer_when_quantisation_is_exact]


@pytest.mark.parametrize("name,attr,val", [
    ("floor exponent (saturating)", "quantize_mx", _mx_scale_floor),
    ("blocks of 32 rows", "MX_BLOCK", (32, 1)),
])
def test_mx_mutant_is_caught(name, attr, val, monkeypatch):
    if attr == "MX_BLOCK":
        def by_rows(W):
            c, s = _orig_mx(np.asarray(W, np.float32).T)
            return c.T.copy(), s.T.copy()
        monkeypatch.setattr(f8, "quantize_mx", by_rows)
    monkeypatch.setattr(f8, attr, val)
    caught = []
    for pin in _MX_PINS:
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches: {name}"
