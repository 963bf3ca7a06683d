"""The PID bias controller: its fp64 oracle against closed forms, the C
library's controller against the oracle, convergence of the zero-expert share
on a stream of batches routed by the oracle, and the cross-rank histogram sum
on a two-process gloo group."""
import os

import numpy as np
import pytest
import torch

from mixture_experts_layer_28_b200 import build as mb
from mixture_experts_layer_28_b200 import moe_zc as mz
from mixture_experts_layer_28_b200 import workloads as wl
from oracle import bias_controller_ref as pc
from oracle import moe_zc_ref as ref


@pytest.fixture(scope="module", autouse=True)
def _lib():
    mb.build()
    mz.lib()


# ---------------------------------------------------------------- oracle pins
def test_oracle_set_point_sums_to_all_picks():
    t = pc.target_load(6, 3, tokens=100, K=4, rho=0.25)
    assert np.isclose(t.sum(), 400.0)
    assert np.allclose(t[:6], 0.75 * 400 / 6) and np.allclose(t[6:], 0.25 * 400 / 3)


def test_oracle_closed_form_step_responses():
    """Constant load error e: P gives kp e, I gives ki n e after n steps, D
    gives kd e on the first step and 0 afterwards; on target nothing moves."""
    N, Z, T, K = 3, 1, 40, 2          # 80 picks, mean load 20
    base = np.array([0.1, -0.2, 0.3, 0.0])
    rho = 0.25                        # targets: 20, 20, 20 | 20
    counts = np.array([10, 30, 20, 20])
    e = np.array([0.5, -0.5, 0.0, 0.0])
    st = pc.PidState(base)
    for n in range(1, 6):
        b = pc.step(st, counts, N, Z, T, K, rho, kp=0.1, ki=0.0, kd=0.0)
        np.testing.assert_allclose(b, base + 0.1 * e, rtol=0, atol=1e-15)
    st = pc.PidState(base)
    for n in range(1, 6):
        b = pc.step(st, counts, N, Z, T, K, rho, kp=0.0, ki=0.01, kd=0.0)
        np.testing.assert_allclose(b, base + 0.01 * n * e, rtol=0, atol=1e-15)
    st = pc.PidState(base)
    b1 = pc.step(st, counts, N, Z, T, K, rho, kp=0.0, ki=0.0, kd=0.2)
    b2 = pc.step(st, counts, N, Z, T, K, rho, kp=0.0, ki=0.0, kd=0.2)
    np.testing.assert_allclose(b1, base + 0.2 * e, atol=1e-15)
    np.testing.assert_allclose(b2, base, atol=1e-15)
    st = pc.PidState(base)
    b = pc.step(st, [20, 20, 20, 20], N, Z, T, K, rho, kp=1.0, ki=1.0, kd=1.0)
    np.testing.assert_allclose(b, base, atol=1e-15)
    st = pc.PidState(base)
    b = pc.step(st, counts, N, Z, T, K, rho, kp=10.0, ki=0.0, kd=0.0, max_shift=0.3)
    np.testing.assert_allclose(b, base + np.clip(10 * e, -0.3, 0.3), atol=1e-15)


def test_oracle_integral_does_not_wind_up_while_clipped():
    """Integral term alone (ki = 0.07), error +-0.5, clip 0.3.  Step n gives
    0.035 n until 0.035 n would pass the clip (n = 9): from then on the
    integral stays at 8 e and the output at 0.28.  After 20 such steps the
    load turns (error -+0.5): the integral drops to 7 e at once and the
    output to 0.245 -- without the remedy the integral would be 20 e and the
    output would stay clipped at 0.3 for another dozen steps."""
    N, Z, T, K = 3, 1, 40, 2
    base = np.array([0.1, -0.2, 0.3, 0.0])
    rho = 0.25
    st = pc.PidState(base)
    for n in range(1, 21):
        b = pc.step(st, [10, 30, 20, 20], N, Z, T, K, rho, kp=0.0, ki=0.07, kd=0.0,
                    max_shift=0.3)
        want = 0.07 * 0.5 * min(n, 8)
        np.testing.assert_allclose(b[:2], base[:2] + np.array([want, -want]), atol=1e-12)
    np.testing.assert_allclose(st.integral[:2], [4.0, -4.0], atol=1e-12)
    b = pc.step(st, [30, 10, 20, 20], N, Z, T, K, rho, kp=0.0, ki=0.07, kd=0.0, max_shift=0.3)
    np.testing.assert_allclose(b[:2], base[:2] + np.array([0.245, -0.245]), atol=1e-12)


def test_library_matches_oracle_through_saturation():
    """The C controller against the oracle over a saturating stretch and a
    turn of the load, with P, I and D all on."""
    N, Z, T, K = 3, 1, 40, 2
    base = np.array([0.1, -0.2, 0.3, 0.0], dtype=np.float32)
    pid = dict(rho=0.25, kp=0.05, ki=0.07, kd=0.02, max_shift=0.3)
    ctl = mz.BiasController(base, N, Z, K, target_zero_frac=pid["rho"], kp=pid["kp"],
                            ki=pid["ki"], kd=pid["kd"], max_shift=pid["max_shift"])
    st = pc.PidState(base.astype(np.float64))
    for n in range(30):
        counts = [10, 30, 20, 20] if n < 20 else [30, 10, 20, 20]
        got = ctl.step(np.array(counts, dtype=np.int32), T)
        want = pc.step(st, counts, N, Z, T, K, pid["rho"], pid["kp"], pid["ki"], pid["kd"],
                       pid["max_shift"])
        np.testing.assert_allclose(got, want, rtol=1e-5, atol=1e-6)


# ---------------------------------------------------------------- C vs oracle
def test_library_controller_matches_oracle():
    rng = np.random.default_rng(0)
    N, Z, K, T = 7, 5, 3, 64
    b0 = rng.uniform(-0.1, 0.1, N + Z).astype(np.float32)
    ctl = mz.BiasController(b0, N, Z, K, target_zero_frac=0.3, kp=0.05, ki=0.01, kd=0.02,
                            max_shift=0.5)
    st = pc.PidState(b0.astype(np.float64))
    for _ in range(12):
        counts = rng.multinomial(T * K, np.ones(N + Z) / (N + Z))
        got = ctl.step(counts, T)
        want = pc.step(st, counts, N, Z, T, K, 0.3, 0.05, 0.01, 0.02, 0.5)
        np.testing.assert_allclose(got, want, rtol=1e-5, atol=1e-6)


def test_library_controller_argument_checks():
    L = mz.lib()
    b = np.zeros(4, np.float32)
    st = np.zeros(12, np.float32)
    c = np.zeros(4, np.int32)
    pid = mz.Pid(0.5, 0.1, 0.0, 0.0, 0.0)
    import ctypes
    step = lambda N, Z, T, K, p=pid: L.moe_zc_bias_controller_step(
        c.ctypes.data, N, Z, T, K, ctypes.byref(p), st.ctypes.data, b.ctypes.data)
    assert step(2, 2, 10, 2) == mz.OK
    assert step(2, 2, 0, 2) == mz.ERR_INVALID_ARG          # no tokens
    assert step(2, 2, 10, 5) == mz.ERR_INVALID_ARG         # K > E
    assert step(4, 0, 10, 2) == mz.ERR_INVALID_ARG         # rho = 0.5 but no zero experts
    assert step(2, 2, 10, 2, mz.Pid(1.5, 0.1, 0, 0, 0)) == mz.ERR_INVALID_ARG
    assert L.moe_zc_bias_controller_init(None, 4, st.ctypes.data) == mz.ERR_INVALID_ARG


# ---------------------------------------------------------------- closed loop
@pytest.mark.parametrize("name,T,rho", [("tiny", 256, 0.1), ("small", 512, 0.5)])
def test_controller_steers_zero_share_on_oracle_routing(name, T, rho):
    """A stream of fresh batches routed by the fp64 oracle; after 60 steps the
    zero-expert share sits at the set-point and FFN load is evened out."""
    w = wl.get(name, T=T)
    ri = wl.routing_inputs(w)
    ctl = mz.BiasController(ri.b0.numpy(), w.N, w.Z, w.K, target_zero_frac=rho,
                            kp=0.01, ki=0.002)
    b = ri.b0.numpy().copy()
    share, imb = [], []
    for s in range(60):
        g = torch.Generator().manual_seed(5000 + s)
        x = torch.randn(T, w.d, generator=g).to(torch.bfloat16)
        r = ref.route(x, ri.W_r, b, w.N, w.K)
        cnt = ref.expert_load(r.idx, w.E)
        share.append(ref.zero_pick_fraction(r.idx, w.N))
        ffn = cnt[: w.N]
        imb.append(ffn.max() / max(ffn.mean(), 1e-9))
        b = ctl.step(cnt, T)
    assert abs(np.mean(share[-10:]) - rho) <= 0.03, (share[0], share[-10:])
    assert abs(share[0] - rho) > 0.15                   # it had somewhere to go
    assert np.mean(imb[-10:]) < 0.5 * imb[0]


# ---------------------------------------------------------------- two ranks
def _allreduce_worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        counts = np.arange(6, dtype=np.int32) * (rank + 1)
        q.put((rank, mz.allreduce_expert_load(counts).tolist()))
    finally:
        dist.destroy_process_group()


def test_expert_load_allreduce_two_ranks():
    import socket
    import torch.multiprocessing as tmp
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = tmp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_allreduce_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=10) for _ in range(2))
    want = (np.arange(6) * 3).tolist()
    assert got[0] == want and got[1] == want
