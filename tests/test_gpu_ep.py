"""The expert-parallel building blocks on the GPU, through the C ABI.

* moe_zc_route -> moe_zc_dispatch -> moe_zc_experts -> moe_zc_combine on
  one device equals moe_zc_forward bit for bit (same router plan, the same
  GEMMs in the same reduction order).
* Two ranks' steps run in lock-step in one process (mixture_experts_layer_28_b200.ep.EpRank,
  the exchange done by copying segments between the two ranks' buffers):
  each rank's output equals moe_zc_forward on its own tokens bit for bit,
  and the summed histograms equal the histogram of both ranks' picks.
* ep.forward on a one-rank NCCL process group equals moe_zc_forward.
(Ranks on separate GPUs are not run: one GPU here.)
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_28_b200 import ep
from mixture_experts_layer_28_b200 import moe_zc as mz
from mixture_experts_layer_28_b200 import workloads as wl
from parity import Case, check_output, check_routing
from oracle import moe_zc_ref as ref

pytestmark = pytest.mark.gpu


def _forward(case, x):
    w, d, ew = case.w, case.dev, case.ew
    out = mz.forward(x, d["W_r"], d["b"], ew.W_gate, ew.W_up, ew.W_down, w.N, w.Z, w.K,
                     logit_offset=d["off"])
    torch.cuda.synchronize()
    mz.synchronize()
    return out


@pytest.mark.parametrize("name,kw", [("small", dict(T=1024)), ("skewed40", dict(T=700, d=512, I=256)),
                                     ("decode", dict(d=1024, I=256))])
def test_steps_on_one_device_equal_forward(name, kw):
    case = Case(wl.get(name, **kw))
    w, d, ew = case.w, case.dev, case.ew
    want = _forward(case, d["x"])
    idx, gate, zsum, counts = mz.route(d["x"], d["W_r"], d["b"], w.N, w.Z, w.K, d["off"])
    rows = int(counts[: w.N].sum().item())
    slot, send, send_expert = mz.dispatch(d["x"], idx, counts, w.N, rows)
    y = mz.experts(send, send_expert, 0, ew.W_gate, ew.W_up, ew.W_down)
    out = mz.combine(d["x"], y, slot, gate, zsum)
    torch.cuda.synchronize()
    mz.synchronize()
    assert torch.equal(out, want)
    # the routing steps against the oracle as in every parity test
    r = case.oracle_routing()
    ok = check_routing(case, r, idx.cpu().numpy(), gate.cpu().numpy(), counts.cpu().numpy())
    np.testing.assert_allclose(zsum.cpu().numpy()[ok], r.zsum[ok], rtol=1e-4, atol=1e-9)
    # packed dispatch: rows grouped by expert, slots a permutation of the FFN picks
    se = send_expert.cpu().numpy()
    assert np.all(np.diff(se) >= 0)
    sl = slot.cpu().numpy()
    ffn = idx.cpu().numpy() < w.N
    assert np.array_equal(np.sort(sl[ffn]), np.arange(rows)) and np.all(sl[~ffn] == -1)


def test_two_ranks_in_lock_step_equal_forward():
    w = wl.get("small", T=900)
    case = Case(w)
    d, ew = case.dev, case.ew
    world = 2
    split = [380, 520]
    xs = list(d["x"].split(split))
    router = ep.Router(d["W_r"], d["b"], d["off"])
    ranks = []
    for r in range(world):
        lo, hi = ep.shard_range(w.N, world, r)
        shard = ep.ExpertShard(lo, ew.W_gate[lo:hi], ew.W_up[lo:hi], ew.W_down[lo:hi])
        ranks.append(ep.EpRank(world, r, w.N, w.Z, w.K, router, shard))
    sends = [rk.prepare(x.contiguous()) for rk, x in zip(ranks, xs)]
    # the exchange: rank j receives, in rank order, every rank's segment j
    segs = [(s.split(sp), se.split(sp)) for s, se, sp in sends]
    results = []
    for j in range(world):
        rows = torch.cat([segs[i][0][j] for i in range(world)])
        expert = torch.cat([segs[i][1][j] for i in range(world)])
        results.append(ranks[j].compute(rows, expert))
    # and back: rank i gets, in its send order, its rows from every rank
    recv_sizes = [[sends[i][2][j] for i in range(world)] for j in range(world)]
    outs = []
    for i in range(world):
        back = torch.cat([results[j].split(recv_sizes[j])[i] for j in range(world)])
        outs.append(ranks[i].finish(back))
    torch.cuda.synchronize()
    mz.synchronize()
    total = torch.zeros(w.E, dtype=torch.int64)
    for i in range(world):
        assert torch.equal(outs[i], _forward(case, xs[i].contiguous())), i
        total += ranks[i].counts.cpu().to(torch.int64)
    mz.forward(d["x"], d["W_r"], d["b"], ew.W_gate, ew.W_up, ew.W_down, w.N, w.Z, w.K,
               logit_offset=d["off"])
    torch.cuda.synchronize()
    idx, _ = mz.last_routing(w.T, w.K)
    near = case.oracle_routing().gap < 1e-5
    # histogram of both ranks = the batch's, away from tokens whose picks are
    # near-ties (the two rank-sized router GEMMs slice the contraction
    # differently from one batch-sized one)
    got = total.numpy() - np.bincount(
        np.concatenate([r.idx.cpu().numpy() for r in ranks])[near].ravel(), minlength=w.E)
    want = np.bincount(idx.ravel(), minlength=w.E) - np.bincount(idx[near].ravel(), minlength=w.E)
    assert np.array_equal(got, want)


def test_process_group_forward_one_rank():
    import torch.distributed as dist
    w = wl.get("small", T=600)
    case = Case(w)
    d, ew = case.dev, case.ew
    store = dist.HashStore()
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        shard = ep.ExpertShard(0, ew.W_gate, ew.W_up, ew.W_down)
        out, counts = ep.forward(d["x"], ep.Router(d["W_r"], d["b"], d["off"]), shard,
                                 w.N, w.Z, w.K)
        torch.cuda.synchronize()
        want = _forward(case, d["x"])
        assert torch.equal(out, want)
        assert np.array_equal(counts.cpu().numpy(), mz.expert_load(w.E))
    finally:
        dist.destroy_process_group()
    # and the output against the oracle, with the parity bounds
    r = case.oracle_routing()
    ok = r.gap >= 1e-5
    out_o = ref.forward_rows(case.x, r, case.expert)
    check_output(out.float().cpu().numpy().astype(np.float64)[ok], out_o[ok])
