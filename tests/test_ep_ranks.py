"""Expert parallelism (mixture_experts_layer_28_b200.ep) on two host ranks
over gloo: each rank routes its own tokens, sends its FFN picks' rows to the
rank owning each expert, computes its expert range on what it receives,
sends the results back and combines; zero-expert picks stay local.  The
compute steps come from the fp64 oracle (tests/ep_oracle_backend.py), so
what is checked here is the exchange: segment sizes, row order both ways,
expert ids, the combine's slots and the exact histogram all-reduce.  Each
rank's output must equal the oracle's single-process forward of its tokens,
and the all-reduced histogram the histogram of all tokens."""
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _layer(case):
    """Small layer: N = 8 FFN experts (4 per rank), Z = 4 zero experts, K = 3."""
    r = np.random.default_rng(21)
    N, Z, K, d, I, T = 8, 4, 3, 16, 12, 40
    E = N + Z
    L = dict(N=N, Z=Z, K=K, x=r.standard_normal((T, d)), W_r=r.standard_normal((E, d)) * 0.3,
             b=r.uniform(-0.1, 0.1, E), W_gate=r.standard_normal((N, I, d)) * 0.3,
             W_up=r.standard_normal((N, I, d)) * 0.3, W_down=r.standard_normal((N, d, I)) * 0.3,
             split=[17, 23])
    if case == "hot_remote":      # rank 0's tokens all pick expert 6 (rank 1's)
        L["b"][6] += 10.0
    elif case == "all_zero_on_rank0":
        L["b"][N:] += 10.0        # every pick a zero expert: no rows travel
    elif case == "uneven":
        L["split"] = [3, 37]
    return L


def _worker(rank, world, port, case, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch
    import torch.distributed as dist
    from ep_oracle_backend import OracleBackend
    from mixture_experts_layer_28_b200 import ep
    from oracle import moe_zc_ref as ref

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        L = _layer(case)
        N, Z, K = L["N"], L["Z"], L["K"]
        t0 = sum(L["split"][:rank])
        x = torch.from_numpy(L["x"][t0:t0 + L["split"][rank]])
        lo, hi = ep.shard_range(N, world, rank)
        shard = ep.ExpertShard(lo, L["W_gate"][lo:hi], L["W_up"][lo:hi], L["W_down"][lo:hi])
        router = ep.Router(torch.from_numpy(L["W_r"]), torch.from_numpy(L["b"]))
        out, counts = ep.forward(x, router, shard, N, Z, K, backend=OracleBackend())
        want, r = ref.forward(x.numpy(), L["W_r"], L["b"], L["W_gate"], L["W_up"], L["W_down"],
                              N, Z, K)
        _, r_all = ref.forward(L["x"], L["W_r"], L["b"], L["W_gate"], L["W_up"], L["W_down"],
                               N, Z, K)
        q.put((rank, float(np.max(np.abs(out.numpy() - want))),
               float(np.max(np.abs(want))) if want.size else 0.0,
               counts.numpy().tolist(), ref.expert_load(r_all.idx, N + Z).tolist(),
               int((r.idx < N).sum())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", ["random", "hot_remote", "all_zero_on_rank0", "uneven"])
def test_two_rank_expert_parallel_forward(case):
    import torch.multiprocessing as tmp
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = tmp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, case, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, err, scale, counts, want_counts, ffn in res:
        assert err <= 1e-12 * (1.0 + scale), (case, rank, err)
        assert counts == want_counts, (case, rank)   # exact all-reduced histogram
    if case == "all_zero_on_rank0":
        assert all(r[5] == 0 for r in res)          # no FFN pick anywhere
    if case == "hot_remote":
        assert res[0][5] > 0


def test_send_splits_follow_expert_ranges():
    sys.path.insert(0, ROOT)
    from mixture_experts_layer_28_b200 import ep
    assert ep.send_splits([3, 0, 5, 1, 2, 2, 0, 7], 2) == [9, 11]
    assert ep.send_splits([3, 0, 5, 1, 2, 2, 0, 7], 4) == [3, 6, 4, 7]
    assert ep.shard_range(8, 4, 3) == (6, 8)
    with pytest.raises(ValueError):
        ep.shard_range(10, 4, 0)
