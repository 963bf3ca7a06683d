"""The C-ABI library loads and exports what include/moe_zc.h declares, and its
host-side argument checks return the documented status codes (no GPU needed:
invalid arguments are rejected before any CUDA call)."""
import ctypes

import pytest
import torch

from mixture_experts_layer_28_b200 import build as mb
from mixture_experts_layer_28_b200 import moe_zc as mz


@pytest.fixture(scope="module")
def L():
    mb.build()
    return mz.lib()


def test_exports_every_declared_symbol(L):
    names = mz.declared_symbols()
    assert "moe_zc_forward" in names and "moe_zc_expert_load" in names
    for n in names:
        assert hasattr(L, n), n


def test_size_limits_match_header():
    text = open(mz.HEADER).read()
    assert f"#define MOE_ZC_MAX_K {mz.MAX_K}" in text
    assert f"#define MOE_ZC_MAX_E {mz.MAX_E}" in text


def test_status_strings(L):
    for code in (mz.OK, mz.ERR_INVALID_ARG, mz.ERR_UNSUPPORTED, mz.ERR_CUDA, mz.ERR_OOM,
                 mz.ERR_TIMEOUT, mz.ERR_NO_RESULT):
        s = mz.status_string(code)
        assert s and s != "unknown status"
    assert mz.status_string(12345) == "unknown status"


FAKE = 1 << 20   # an aligned, never-dereferenced address


def _fwd(L, x=FAKE, W_r=FAKE, b=FAKE, Wg=FAKE, Wu=FAKE, Wd=FAKE, T=16, d=128, N=4, Z=2, K=2,
         I=128, out=FAKE):
    return L.moe_zc_forward(x, W_r, b, Wg, Wu, Wd, T, d, N, Z, K, I, out, None)


@pytest.mark.parametrize("kw,status", [
    (dict(x=None), mz.ERR_INVALID_ARG),
    (dict(W_r=None), mz.ERR_INVALID_ARG),
    (dict(out=None), mz.ERR_INVALID_ARG),
    (dict(b=None), mz.ERR_INVALID_ARG),
    (dict(K=0), mz.ERR_INVALID_ARG),
    (dict(K=7), mz.ERR_INVALID_ARG),              # K > E = 6
    (dict(T=-1), mz.ERR_INVALID_ARG),
    (dict(N=-1), mz.ERR_INVALID_ARG),
    (dict(N=0, Z=0, K=1), mz.ERR_INVALID_ARG),    # empty expert pool
    (dict(Wg=None), mz.ERR_INVALID_ARG),          # FFN experts need weights
    (dict(I=0), mz.ERR_INVALID_ARG),
    (dict(d=96), mz.ERR_UNSUPPORTED),             # d % 64
    (dict(d=200), mz.ERR_UNSUPPORTED),
    (dict(I=64), mz.ERR_UNSUPPORTED),             # I % 128
    (dict(N=40, Z=0, K=33), mz.ERR_UNSUPPORTED),  # K > 32
    (dict(N=1000, Z=100, K=2), mz.ERR_UNSUPPORTED),  # E > 1024
    (dict(N=1000, Z=25, K=2), mz.ERR_UNSUPPORTED),   # E = 1025, one past the largest
    (dict(x=FAKE + 8), mz.ERR_UNSUPPORTED),       # misaligned
    (dict(Wd=FAKE + 2), mz.ERR_UNSUPPORTED),
])
def test_argument_checks(L, kw, status):
    assert _fwd(L, **kw) == status


# The next checks pass the argument checks with fake pointers, so the call
# goes on to the device: run them only where there is none.
_no_device = pytest.mark.skipif(torch.cuda.is_available(),
                                reason="fake pointers must not reach a GPU")


@_no_device
def test_zero_ffn_experts_need_no_weights(L):
    # N = 0: weights may be NULL and I is ignored; only the device call can fail here
    st = _fwd(L, Wg=None, Wu=None, Wd=None, N=0, Z=4, K=2, I=0)
    assert st in (mz.OK, mz.ERR_CUDA, mz.ERR_UNSUPPORTED)


@_no_device
@pytest.mark.parametrize("d", [64, 192, 320])
def test_widths_of_whole_k_steps_are_accepted(L, d):
    """d needs only whole 64-wide contraction steps (d % 64 == 0); the
    down projection's last 128-row weight block may be half past d."""
    assert _fwd(L, d=d) == mz.ERR_CUDA   # past the checks; no device here


def _noalloc(L, status=FAKE, d=128, **kw):
    a = dict(x=FAKE, W_r=FAKE, b=FAKE, off=None, T=16, N=4, Z=2, K=2, idx=FAKE, gate=FAKE,
             counts=FAKE)
    a.update(kw)
    return L.moe_zc_route_noalloc(a["x"], a["W_r"], a["b"], a["off"], a["T"], d, a["N"], a["Z"],
                                  a["K"], a["idx"], a["gate"], a["counts"], status, None)


def test_noalloc_argument_checks(L):
    assert _noalloc(L, status=None) == mz.ERR_INVALID_ARG   # the status word is required
    assert _noalloc(L, counts=None) == mz.ERR_INVALID_ARG
    assert _noalloc(L, d=96) == mz.ERR_UNSUPPORTED
    assert _noalloc(L, T=1364, N=512, Z=256, K=12) == mz.ERR_UNSUPPORTED   # past the array


def test_reserve_argument_checks(L):
    assert L.moe_zc_reserve(-1, 128, 4, 2, 2, 128) == mz.ERR_INVALID_ARG
    assert L.moe_zc_reserve(16, 128, 4, 2, 0, 128) == mz.ERR_INVALID_ARG
    assert L.moe_zc_reserve(16, 128, 0, 0, 1, 128) == mz.ERR_INVALID_ARG


def test_host_queries_reject_null(L):
    assert L.moe_zc_expert_load(None) == mz.ERR_INVALID_ARG
    assert L.moe_zc_last_expert(0, 4, None, None, None, None) == mz.ERR_INVALID_ARG


def test_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros(16, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        mz.forward(x, torch.zeros(6, 128, dtype=torch.bfloat16), torch.zeros(6), None, None, None,
                   N=0, Z=6, K=2)


def test_fp8_entry_points_argument_checks(L):
    f = FAKE
    fwd8 = lambda **kw: L.moe_zc_forward_fp8(
        kw.get("x", f), f, f, kw.get("wg", f), kw.get("wg_sf", f), kw.get("wu", f),
        kw.get("wu_sf", f), f, 16, kw.get("d", 256), 4, 2, 2, 128, None, f, None)
    assert fwd8(wg_sf=None) == mz.ERR_INVALID_ARG           # scales are required
    assert fwd8(wu_sf=None) == mz.ERR_INVALID_ARG
    assert fwd8(d=192) == mz.ERR_UNSUPPORTED                # 128 contraction elements a stage
    assert fwd8(wg_sf=f + 4) == mz.ERR_UNSUPPORTED          # misaligned scales
    q = L.moe_zc_fp8_quantize_weights
    assert q(None, 128, 128, f, f, None) == mz.ERR_INVALID_ARG
    assert q(f, 0, 128, f, f, None) == mz.ERR_INVALID_ARG
    assert q(f, 130, 128, f, f, None) == mz.ERR_UNSUPPORTED  # rows % 128
    assert q(f, 128, 96, f, f, None) == mz.ERR_UNSUPPORTED   # cols % 128
    assert q(f, 128, 128, f + 8, f, None) == mz.ERR_UNSUPPORTED


def test_expert_parallel_steps_argument_checks(L):
    f = FAKE
    # moe_zc_route: as the forward's router arguments
    r = lambda **kw: L.moe_zc_route(f, f, f, None, kw.get("T", 16), kw.get("d", 128), 4, 2,
                                    kw.get("K", 2), f, f, f, kw.get("counts", f), None)
    assert r(counts=None) == mz.ERR_INVALID_ARG
    assert r(K=0) == mz.ERR_INVALID_ARG
    assert r(d=96) == mz.ERR_UNSUPPORTED
    # moe_zc_dispatch
    dsp = lambda **kw: L.moe_zc_dispatch(kw.get("x", f), f, f, 16, kw.get("d", 128),
                                         kw.get("N", 4), 2, f, kw.get("send", f), f, None)
    assert dsp(N=0) == mz.ERR_INVALID_ARG
    assert dsp(send=None) == mz.ERR_INVALID_ARG
    assert dsp(d=100) == mz.ERR_UNSUPPORTED
    assert dsp(x=f + 2) == mz.ERR_UNSUPPORTED
    # moe_zc_experts: given routing of R rows over N local experts
    ex = lambda **kw: L.moe_zc_experts(f, kw.get("expert", f), 0, 16, kw.get("d", 128),
                                       kw.get("N", 4), 128, f, f, f, f, None)
    assert ex(expert=None) == mz.ERR_INVALID_ARG
    assert ex(N=0) == mz.ERR_INVALID_ARG
    assert ex(d=96) == mz.ERR_UNSUPPORTED
    # moe_zc_combine
    cb = lambda **kw: L.moe_zc_combine(kw.get("x", f), f, f, f, f, 16, kw.get("d", 128),
                                       kw.get("K", 2), f, None)
    assert cb(x=None) == mz.ERR_INVALID_ARG
    assert cb(K=0) == mz.ERR_INVALID_ARG
    assert cb(d=100) == mz.ERR_UNSUPPORTED
