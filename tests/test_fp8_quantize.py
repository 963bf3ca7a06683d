"""The library's host FP8 quantiser (moe_zc_fp8_quantize) against the FP8
oracle, code for code and scale for scale, in both block readings; no GPU."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_28_b200 import build as mb
from mixture_experts_layer_28_b200 import moe_zc as mz
from oracle import fp8_ref as f8


@pytest.fixture(scope="module", autouse=True)
def _lib():
    mb.build()
    mz.lib()


def _oracle(W, mode):
    Wf = W.float().numpy()
    return f8.quantize_weight(Wf) if mode == mz.FP8_BLOCK128 else f8.quantize_mx(Wf)


def _cases():
    g = torch.Generator().manual_seed(0)
    yield "gaussian", (torch.randn(256, 384, generator=g) * 0.02).to(torch.bfloat16)
    yield "ragged", (torch.randn(200, 301, generator=g) * 3.0).to(torch.bfloat16)
    w = (torch.randn(130, 160, generator=g) * 1e-3).to(torch.bfloat16)
    w[:, :40] = 0.0                                   # all-zero blocks
    w[7, 50] = 1e-30                                   # tiny: subnormal codes
    yield "zeros and tiny", w
    # wide magnitudes: every block holds values across the subnormal range
    e = torch.randint(-40, 10, (128, 256), generator=g).float()
    yield "wide exponents", (torch.sign(torch.randn(128, 256, generator=g)) * 2.0 ** e).to(torch.bfloat16)
    w = (torch.randn(128, 128, generator=g)).to(torch.bfloat16)
    w[3, 3] = float("nan")
    w[100, 5] = float("inf")
    yield "non-finite", w


@pytest.mark.parametrize("mode", [mz.FP8_BLOCK128, mz.FP8_MX32])
def test_matches_oracle_bit_for_bit(mode):
    for name, W in _cases():
        codes, scales = mz.fp8_quantize(W, mode)
        oc, os_ = _oracle(W, mode)
        assert np.array_equal(scales, os_), name
        assert np.array_equal(codes, oc), (name, int((codes != oc).sum()))


def test_ties_and_saturation_boundaries():
    # one 128 x 128 block (2 x 128 here) whose maximum is 448 (scale 1): row 0
    # holds every midpoint between neighbouring E4M3 values (ties: to the
    # even code), row 1 every E4M3 value itself
    pos = f8.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mids = (pos[:-1] + pos[1:]) / 2
    W = np.zeros((2, 128), dtype=np.float32)
    W[0, : mids.size] = mids
    W[0, 127] = 448.0
    W[1, : pos.size] = pos
    Wt = torch.from_numpy(W).to(torch.bfloat16)
    keep = Wt.float().numpy() == W                   # bf16-representable entries
    assert keep[1].all()
    for mode in (mz.FP8_BLOCK128, mz.FP8_MX32):
        codes, scales = mz.fp8_quantize(Wt, mode)
        oc, _ = _oracle(Wt, mode)
        assert np.array_equal(codes, oc)
        if mode == mz.FP8_BLOCK128:
            assert scales.shape == (1, 1) and scales[0, 0] == 1.0
            assert codes[0, 127] == 0x7E and np.array_equal(codes[1, :127], np.arange(127))
            assert np.array_equal(codes[keep], f8.e4m3_encode(W[keep]))
            ties = keep[0, : mids.size]
            assert np.all(codes[0, : mids.size][ties] % 2 == 0)


def test_argument_checks():
    L = mz.lib()
    buf = np.zeros(16, dtype=np.uint8)
    sc = np.zeros(4, dtype=np.float32)
    W = torch.zeros(2, 2, dtype=torch.bfloat16)
    assert L.moe_zc_fp8_quantize(None, 2, 2, 0, buf.ctypes.data, sc.ctypes.data) == mz.ERR_INVALID_ARG
    assert L.moe_zc_fp8_quantize(W.data_ptr(), 0, 2, 0, buf.ctypes.data, sc.ctypes.data) == mz.ERR_INVALID_ARG
    assert L.moe_zc_fp8_quantize(W.data_ptr(), 2, 2, 7, buf.ctypes.data, sc.ctypes.data) == mz.ERR_INVALID_ARG
    with pytest.raises(ValueError):
        mz.fp8_quantize(torch.zeros(4, dtype=torch.bfloat16))
