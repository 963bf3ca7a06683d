"""The forward captured once into a CUDA graph (the stream capture a caller
does to cut per-call launch cost at decode) and replayed: the replay matches
the eager call bit for bit, and after new token values are written into the
captured input buffer a replay matches an eager forward on those values."""
import pytest
import torch

from mixture_experts_layer_28_b200 import build as mb
from mixture_experts_layer_28_b200 import moe_zc as mz
from mixture_experts_layer_28_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    mb.build()
    mz.lib()


@pytest.mark.parametrize("name,over", [
    ("small", dict(T=512)),
    ("decode", dict(N=48, Z=24)),            # decode-shaped: 64 tokens, K slices in the router
    ("skewed40", dict(T=1024, d=512, I=256)),  # logit offset
])
def test_forward_replays_from_cuda_graph(name, over):
    w = wl.get(name, **over)
    ri = wl.routing_inputs(w)
    ew = wl.expert_weights(w, "cuda")
    x = ri.x.cuda()
    W_r = ri.W_r.cuda()
    b = ri.bias(w.N, w.delta).cuda()
    off = None if ri.logit_offset is None else ri.logit_offset.cuda()
    args = (W_r, b, ew.W_gate, ew.W_up, ew.W_down, w.N, w.Z, w.K)

    # the workspace is sized before the capture, which then allocates nothing
    mz.reserve(w.T, w.d, w.N, w.Z, w.K, w.I)
    ref = mz.forward(x, *args, logit_offset=off)
    torch.cuda.synchronize()
    load_ref = mz.expert_load(w.E)

    out = torch.empty_like(x)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        mz.forward(x, *args, out=out, logit_offset=off)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    assert (mz.expert_load(w.E) == load_ref).all()

    gen = torch.Generator().manual_seed(77)
    x2 = torch.randn(w.T, w.d, generator=gen).to(torch.bfloat16).cuda()
    x.copy_(x2)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    replayed = out.clone()
    load_replayed = mz.expert_load(w.E)
    ref2 = mz.forward(x2, *args, logit_offset=off)
    torch.cuda.synchronize()
    assert torch.equal(replayed, ref2)
    assert (load_replayed == mz.expert_load(w.E)).all()
    assert not torch.equal(ref2, ref)
    del g
