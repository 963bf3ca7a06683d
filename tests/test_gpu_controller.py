"""Closed loop on the GPU: forward through the C ABI, histogram from
moe_zc_expert_load, new biases from the library's PID controller, next
forward -- the zero-expert share settles at the set-point."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_28_b200 import moe_zc as mz
from mixture_experts_layer_28_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def test_controller_steers_gpu_forward():
    w = wl.get("small", T=512)
    ri = wl.routing_inputs(w)
    ew = wl.expert_weights(w, "cuda")
    W_r = ri.W_r.cuda()
    rho = 0.5
    ctl = mz.BiasController(ri.b0.numpy(), w.N, w.Z, w.K, target_zero_frac=rho,
                            kp=0.01, ki=0.002)
    b = ri.b0.clone()
    share = []
    for s in range(50):
        g = torch.Generator().manual_seed(7000 + s)
        x = torch.randn(w.T, w.d, generator=g).to(torch.bfloat16).cuda()
        mz.forward(x, W_r, b.cuda(), ew.W_gate, ew.W_up, ew.W_down, w.N, w.Z, w.K)
        cnt = mz.expert_load(w.E)                   # waits for the forward
        assert cnt.sum() == w.T * w.K
        share.append(float(cnt[w.N:].sum()) / (w.T * w.K))
        b = torch.from_numpy(ctl.step(cnt, w.T))
    assert abs(share[0] - rho) > 0.15
    assert abs(np.mean(share[-10:]) - rho) <= 0.03, share[-10:]
