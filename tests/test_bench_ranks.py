"""bench.py's multi-rank plumbing on two host-only ranks (gloo): the world size
check, the barrier and the max-over-ranks reduction of step times."""
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world), CUDA_VISIBLE_DEVICES="")
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist(world)
    try:
        d.barrier()
        q.put((rank, d.max(10.0 + rank), d.rank, d.world))
    finally:
        d.close()


def test_two_host_ranks_take_the_slowest_time():
    import torch.multiprocessing as tmp
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = tmp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert [g[1] for g in got] == [11.0, 11.0]
    assert [(g[2], g[3]) for g in got] == [(0, 2), (1, 2)]


def test_world_size_must_match_gpus(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "1")
    with pytest.raises(SystemExit):
        bench.Dist(2)
