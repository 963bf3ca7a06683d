"""moe_zc_plan: the launch decisions a forward takes, checked on the host
(no GPU): the router GEMM's tiling, and whether a small batch runs the rest
of the forward (route, dispatch, both expert GEMMs, combine) in one
persistent grid or falls back to separate launches."""
import pytest

from mixture_experts_layer_28_b200 import build as mb
from mixture_experts_layer_28_b200 import moe_zc as mz

DECODE = dict(T=64, d=6144, N=512, Z=256, K=12, I=2048)
PREFILL = dict(DECODE, T=16384)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    mb.build()
    mz.lib()
    yield
    mz.test_one_grid(False)


def test_decode_runs_expert_gemms_in_one_grid():
    p = mz.plan(**DECODE, sms=148, resident_blocks=148)
    # the router GEMM and the one grid
    assert p["expert_gemms_one_grid"] == 1 and p["one_grid_step"] == 1 and p["kernels"] == 2
    # tile bound: ceil(64*12/256) + 512 = 515 token tiles; 16 gate/up and 24
    # down weight blocks each -> far more tiles than SMs
    assert p["expert_grid"] == 148
    # 64 tokens are one token tile: six single 128-row blocks of W_r, the
    # contraction sliced 24 ways (96 steps of 64, at least 4 per slice)
    assert p["router_k_slices"] == 24 and p["router_grid"] == 144


def test_one_grid_falls_back_when_not_resident():
    """Fewer resident blocks than the grid needs: two launches instead."""
    p = mz.plan(**DECODE, sms=148, resident_blocks=147)
    assert p["expert_gemms_one_grid"] == 0 and p["one_grid_step"] == 0 and p["kernels"] == 7
    assert p["expert_grid"] == 148       # the gate/up launch
    p = mz.plan(**DECODE, sms=148, resident_blocks=0)   # kernel cannot be resident at all
    assert p["expert_gemms_one_grid"] == 0


def test_one_grid_only_for_small_batches():
    assert mz.plan(**dict(DECODE, T=65))["expert_gemms_one_grid"] == 0
    assert mz.plan(**dict(DECODE, T=1))["expert_gemms_one_grid"] == 1
    p = mz.plan(**PREFILL)
    assert p["expert_gemms_one_grid"] == 0 and p["one_grid_step"] == 0 and p["kernels"] == 7
    # 16384 tokens, E = 768 in 3 paired blocks: 176-token tiles fill two whole
    # waves (282 tiles) where 256-token tiles would leave the second a third full
    assert p["router_token_tile"] == 176 and p["router_k_slices"] == 1
    assert p["router_grid"] == 148


def test_one_grid_test_hook():
    mz.test_one_grid(True)
    try:
        p = mz.plan(**DECODE)
        assert p["expert_gemms_one_grid"] == 0 and p["kernels"] == 7
        # the expert GEMMs in one grid, route, dispatch and combine apart
        mz.test_one_grid(step=False)
        p = mz.plan(**DECODE)
        assert p["expert_gemms_one_grid"] == 1 and p["one_grid_step"] == 0 and p["kernels"] == 6
    finally:
        mz.test_one_grid(False)
    p = mz.plan(**DECODE)
    assert p["expert_gemms_one_grid"] == 1 and p["one_grid_step"] == 1 and p["kernels"] == 2


def test_kernel_counts_of_special_batches():
    assert mz.plan(**dict(DECODE, N=0, Z=768))["kernels"] == 4   # no FFN experts
    assert mz.plan(**dict(DECODE, T=0))["kernels"] == 0


def test_plan_argument_checks():
    with pytest.raises(mz.MoeZcError) as ei:
        mz.plan(**dict(DECODE, d=96))
    assert ei.value.status == mz.ERR_UNSUPPORTED
    with pytest.raises(mz.MoeZcError) as ei:
        mz.plan(**DECODE, sms=0)
    assert ei.value.status == mz.ERR_INVALID_ARG
