"""moe_zc_route_noalloc: the routing stage for callers that cannot let the
library allocate device memory (a server that owns all device memory through
its own pool, a process under a hard memory cap).  Its scratch is a fixed
array inside the library, so this test checks, through the C ABI, that two
calls in a row give the same routing as moe_zc_forward on the same inputs
(picks and histogram exactly, gates within the parity tests' rtol 1e-4), that
the second call leaves the device's free memory unchanged, and that sizes
beyond the array are refused with a clear status.

The file name sorts last so that a run stopping at the first failure has
already run every other test.
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_28_b200 import moe_zc as mz
from mixture_experts_layer_28_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _reference_routing(w, ri, b, ew, off):
    """Routing of the allocating entry point, moe_zc_forward(_ex)."""
    mz.forward(ri.x.cuda(), ri.W_r.cuda(), b.cuda(), ew.W_gate, ew.W_up, ew.W_down,
               w.N, w.Z, w.K, logit_offset=off)
    torch.cuda.synchronize()
    mz.synchronize()
    idx, gate = mz.last_routing(w.T, w.K)
    return idx, gate, mz.expert_load(w.E)


@pytest.mark.parametrize("name,kw", [
    ("small", dict(T=1024)),                       # E = 96
    ("skewed40", dict(T=600, d=512, I=256)),       # E = 384, Zipf logit offset
    ("decode", dict(d=1024, I=256)),               # E = 768, T = 64
])
def test_noalloc_routing_matches_forward(name, kw):
    w = wl.get(name, **kw)
    ri = wl.routing_inputs(w)
    b = ri.bias(w.N, w.delta)
    ew = wl.expert_weights(w, "cuda")
    off = None if ri.logit_offset is None else ri.logit_offset.cuda()
    idx_ref, gate_ref, cnt_ref = _reference_routing(w, ri, b, ew, off)

    x, W_r, bd = ri.x.cuda(), ri.W_r.cuda(), b.cuda()
    idx = torch.empty(w.T, w.K, dtype=torch.int32, device="cuda")
    gate = torch.empty(w.T, w.K, dtype=torch.float32, device="cuda")
    counts = torch.full((w.E,), -7, dtype=torch.int32, device="cuda")   # must be cleared
    status = torch.full((1,), 5, dtype=torch.int32, device="cuda")      # must be cleared
    for call in range(2):
        idx.fill_(-1)
        gate.fill_(-1.0)
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        mz.route_noalloc(x, W_r, bd, w.N, w.Z, w.K, idx, gate, counts,
                         logit_offset=off, status=status)
        torch.cuda.synchronize()
        if call == 1:
            assert torch.cuda.mem_get_info()[0] == free_before, "second call allocated memory"
        assert int(status.item()) == 0
        assert np.array_equal(idx.cpu().numpy(), idx_ref), f"call {call}: picks differ"
        assert np.array_equal(counts.cpu().numpy(), cnt_ref), f"call {call}: histogram differs"
        np.testing.assert_allclose(gate.cpu().numpy(), gate_ref, rtol=1e-4, atol=1e-9)


def test_noalloc_rejects_sizes_beyond_its_array():
    w = wl.get("decode", d=128, I=128)
    T = 1364                                   # one token past the limit at E = 768
    x = torch.zeros(T, w.d, dtype=torch.bfloat16, device="cuda")
    W_r = torch.zeros(w.E, w.d, dtype=torch.bfloat16, device="cuda")
    b = torch.zeros(w.E, dtype=torch.float32, device="cuda")
    idx = torch.empty(T, w.K, dtype=torch.int32, device="cuda")
    gate = torch.empty(T, w.K, dtype=torch.float32, device="cuda")
    counts = torch.empty(w.E, dtype=torch.int32, device="cuda")
    with pytest.raises(mz.MoeZcError) as ei:
        mz.route_noalloc(x, W_r, b, w.N, w.Z, w.K, idx, gate, counts)
    assert ei.value.status == mz.ERR_UNSUPPORTED
    # one token fewer fits
    mz.route_noalloc(x[:1363].contiguous(), W_r, b, w.N, w.Z, w.K, idx[:1363], gate[:1363],
                     counts)
    torch.cuda.synchronize()
    assert int(counts.sum().item()) == 1363 * w.K
