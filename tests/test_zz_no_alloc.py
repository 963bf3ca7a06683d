"""moe_zc_route_noalloc: the routing stage for callers that cannot let the
library allocate device memory (a server that owns all device memory through
its own pool, a process under a hard memory cap).  Its scratch is a fixed
array inside the library.  Through the C ABI, this file checks that

  * two calls in a row route like the fp64 oracle (exact picks and histogram
    away from near-ties, valid top-K at them, gates within rtol 1e-4: the
    tolerances of every GPU parity test) and like moe_zc_forward on the same
    inputs (equal picks and histogram on the tokens that are not near-ties,
    gates within rtol 1e-4);
  * the second call leaves the device's free memory unchanged;
  * sizes beyond the array are refused with a clear status;
  * a bounded device wait that runs out is reported in the caller's status
    word, and the next call is correct again.

The file name sorts last so that a run stopping at the first failure has
already run every other test.
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_28_b200 import moe_zc as mz
from mixture_experts_layer_28_b200 import workloads as wl
from parity import TIE, Case, check_routing

pytestmark = pytest.mark.gpu


def _forward_routing(case):
    """Routing of the allocating entry point, moe_zc_forward(_ex)."""
    case.run()
    torch.cuda.synchronize()
    mz.synchronize()
    idx, gate = mz.last_routing(case.T, case.w.K)
    return idx, gate, mz.expert_load(case.w.E)


def _buffers(case):
    w = case.w
    idx = torch.empty(case.T, w.K, dtype=torch.int32, device="cuda")
    gate = torch.empty(case.T, w.K, dtype=torch.float32, device="cuda")
    counts = torch.full((w.E,), -7, dtype=torch.int32, device="cuda")   # must be cleared
    status = torch.full((1,), 5, dtype=torch.int32, device="cuda")      # must be cleared
    return idx, gate, counts, status


def _noalloc(case, idx, gate, counts, status):
    d, w = case.dev, case.w
    mz.route_noalloc(d["x"], d["W_r"], d["b"], w.N, w.Z, w.K, idx, gate, counts, status,
                     logit_offset=d["off"])


@pytest.mark.parametrize("name,kw", [
    ("small", dict(T=1024)),                       # E = 96
    ("skewed40", dict(T=600, d=512, I=256)),       # E = 384, Zipf logit offset
    ("decode", dict(d=1024, I=256)),               # E = 768, T = 64
])
def test_noalloc_routing_matches_oracle_and_forward(name, kw):
    case = Case(wl.get(name, **kw))
    w = case.w
    r = case.oracle_routing()
    far = r.gap >= TIE
    idx_f, gate_f, cnt_f = _forward_routing(case)
    near = ~far
    cnt_f_far = cnt_f - np.bincount(idx_f[near].ravel(), minlength=w.E)

    idx, gate, counts, status = _buffers(case)
    for call in range(2):
        idx.fill_(-1)
        gate.fill_(-1.0)
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        _noalloc(case, idx, gate, counts, status)
        torch.cuda.synchronize()
        if call == 1:
            assert torch.cuda.mem_get_info()[0] == free_before, "second call allocated memory"
        assert int(status.item()) == 0, f"call {call}: device wait timed out"
        idx_n, gate_n, cnt_n = idx.cpu().numpy(), gate.cpu().numpy(), counts.cpu().numpy()
        # against the oracle, with the parity tests' tolerances
        check_routing(case, r, idx_n, gate_n, cnt_n)
        # against moe_zc_forward on the tokens that are not near-ties
        assert np.array_equal(np.sort(idx_n[far], 1), np.sort(idx_f[far], 1)), f"call {call}"
        cnt_n_far = cnt_n - np.bincount(idx_n[near].ravel(), minlength=w.E)
        assert np.array_equal(cnt_n_far, cnt_f_far), f"call {call}: histogram differs"
        gn = np.take_along_axis(gate_n, np.argsort(idx_n, 1), 1)[far]
        gf = np.take_along_axis(gate_f, np.argsort(idx_f, 1), 1)[far]
        np.testing.assert_allclose(gn, gf, rtol=1e-4, atol=1e-9)


def test_noalloc_reports_a_device_timeout():
    """Every bounded wait of one call limited to 1 ns: the router GEMM gives
    up, the caller's status word says so, and the next call is correct."""
    case = Case(wl.get("small", T=512))
    idx, gate, counts, status = _buffers(case)
    _noalloc(case, idx, gate, counts, status)           # first call: set-up, normal waits
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    mz.test_inject(0, 1)
    _noalloc(case, idx, gate, counts, status)
    torch.cuda.synchronize()
    assert int(status.item()) != 0, "a timed-out wait was not reported"
    _noalloc(case, idx, gate, counts, status)           # the limit applied to one call only
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    check_routing(case, case.oracle_routing(), idx.cpu().numpy(), gate.cpu().numpy(),
                  counts.cpu().numpy())


def test_noalloc_rejects_sizes_beyond_its_array():
    w = wl.get("decode", d=128, I=128)
    T = 1364                                   # one token past the limit at E = 768
    x = torch.zeros(T, w.d, dtype=torch.bfloat16, device="cuda")
    W_r = torch.zeros(w.E, w.d, dtype=torch.bfloat16, device="cuda")
    b = torch.zeros(w.E, dtype=torch.float32, device="cuda")
    idx = torch.empty(T, w.K, dtype=torch.int32, device="cuda")
    gate = torch.empty(T, w.K, dtype=torch.float32, device="cuda")
    counts = torch.empty(w.E, dtype=torch.int32, device="cuda")
    status = torch.empty(1, dtype=torch.int32, device="cuda")
    with pytest.raises(mz.MoeZcError) as ei:
        mz.route_noalloc(x, W_r, b, w.N, w.Z, w.K, idx, gate, counts, status)
    assert ei.value.status == mz.ERR_UNSUPPORTED
    # one token fewer fits
    mz.route_noalloc(x[:1363].contiguous(), W_r, b, w.N, w.Z, w.K, idx[:1363], gate[:1363],
                     counts, status)
    torch.cuda.synchronize()
    assert int(counts.sum().item()) == 1363 * w.K and int(status.item()) == 0
