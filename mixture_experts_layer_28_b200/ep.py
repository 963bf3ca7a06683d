"""Expert parallelism across ranks for the MoE layer with zero-computation
experts.

LongCat-Flash write-up ("Meituan's large model goes viral for its speed"):
section "Shortcut-connected MoE" places the expert computation between a
dispatch and a combine communication step, and section "System-level
optimisation" runs the experts spread over many GPUs.  Here the N FFN
experts are split into R contiguous ranges of N / R, one per rank; the
router, the expert bias and the zero-computation experts are replicated, so a
pick of a zero expert never leaves its rank (it is folded into zsum by the
router), which shrinks the dispatch by the zero-pick share.

One forward on rank r, all compute in the C-ABI library's kernels:

  route      moe_zc_route: picks, gates, zero-gate sums, histogram
  dispatch   moe_zc_dispatch: the FFN picks' rows packed by expert, so the
             rows for rank j's experts are one contiguous segment
  exchange   the segment sizes (all-to-all of R counts), then the rows and
             their expert ids (all-to-all-v)
  experts    moe_zc_experts on the received rows with the local expert range
  exchange   the result rows back, in the order received
  combine    moe_zc_combine: out_t = zsum_t x_t + sum_k g_{t,k} Y[slot_{t,k}]

plus an exact int32 all-reduce of the histogram for the bias controller.
torch.distributed only moves bytes (`all_to_all_single`; NCCL between GPUs,
gloo between host processes).  The sizes of the row exchange are read back
to the host once per forward (the histogram's FFN part, N ints).

The steps are methods of `EpRank`, so that a caller -- or a test -- can run
several ranks' steps in lock-step in one process with its own exchange; the
SPMD `forward` wires them to a process group.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional, Sequence

import torch


@dataclass
class Router:
    """Replicated router: W_r [E, d] bf16, b [E] fp32, optional logit offset."""
    W_r: torch.Tensor
    b: torch.Tensor
    logit_offset: Optional[torch.Tensor] = None


@dataclass
class ExpertShard:
    """FFN experts [base, base + n) of this rank: W_gate, W_up [n, I, d],
    W_down [n, d, I], bf16."""
    base: int
    W_gate: torch.Tensor
    W_up: torch.Tensor
    W_down: torch.Tensor

    @property
    def n(self) -> int:
        return int(self.W_gate.shape[0])


def shard_range(N: int, world: int, rank: int):
    """The FFN experts [lo, hi) rank `rank` owns (contiguous, N % world == 0)."""
    if world < 1 or N % world != 0:
        raise ValueError(f"N = {N} FFN experts do not split evenly over {world} ranks")
    n = N // world
    return rank * n, (rank + 1) * n


def send_splits(counts_ffn: Sequence[int], world: int) -> List[int]:
    """Rows for each rank: the FFN histogram summed over each rank's experts
    (the dispatch packs rows by expert, so these are contiguous segments)."""
    N = len(counts_ffn)
    n = N // world
    return [int(sum(counts_ffn[j * n:(j + 1) * n])) for j in range(world)]


class Library:
    """The compute steps, on the C-ABI library's kernels (CUDA tensors)."""

    def __init__(self):
        from . import moe_zc as mz
        self.mz = mz

    def route(self, x, router: Router, N, Z, K):
        return self.mz.route(x, router.W_r, router.b, N, Z, K, router.logit_offset)

    def dispatch(self, x, idx, counts, N, rows):
        return self.mz.dispatch(x, idx, counts, N, rows)

    def experts(self, rows, expert, shard: ExpertShard):
        return self.mz.experts(rows, expert, shard.base, shard.W_gate, shard.W_up, shard.W_down)

    def combine(self, x, y_rows, slot, gate, zsum):
        return self.mz.combine(x, y_rows, slot, gate, zsum)

    def empty_rows(self, n, like):
        return torch.empty(n, *like.shape[1:], dtype=like.dtype, device=like.device)


class EpRank:
    """One rank's state through the steps of an expert-parallel forward."""

    def __init__(self, world: int, rank: int, N: int, Z: int, K: int, router: Router,
                 shard: ExpertShard, backend=None):
        lo, hi = shard_range(N, world, rank)
        if shard.base != lo or shard.n != hi - lo:
            raise ValueError(f"rank {rank} must own experts [{lo}, {hi})")
        self.world, self.rank, self.N, self.Z, self.K = world, rank, N, Z, K
        self.router, self.shard = router, shard
        self.be = backend if backend is not None else Library()

    # step 1: route and dispatch; returns the rows to send and their sizes
    def prepare(self, x: torch.Tensor):
        self.x = x
        self.idx, self.gate, self.zsum, self.counts = self.be.route(x, self.router, self.N,
                                                                   self.Z, self.K)
        ffn = [int(c) for c in self.counts[: self.N].tolist()]   # the one host read-back
        self.send_splits = send_splits(ffn, self.world)
        self.slot, send, send_expert = self.be.dispatch(x, self.idx, self.counts, self.N,
                                                        sum(self.send_splits))
        return send, send_expert, self.send_splits

    # step 2: the rows received from every rank (in rank order) -> result rows
    def compute(self, rows: torch.Tensor, expert: torch.Tensor):
        return self.be.experts(rows, expert, self.shard)

    # step 3: the result rows of this rank's own picks, back in send order
    def finish(self, y_back: torch.Tensor):
        return self.be.combine(self.x, y_back, self.slot, self.gate, self.zsum)


def forward(x: torch.Tensor, router: Router, shard: ExpertShard, N: int, Z: int, K: int,
            group=None, backend=None):
    """SPMD expert-parallel forward on this rank's tokens x; returns
    (out [T, d], the histogram of all ranks' picks, int32 [E])."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    ep = EpRank(world, rank, N, Z, K, router, shard, backend)
    send, send_expert, splits = ep.prepare(x)
    # segment sizes: what every rank sends to every other
    dev = x.device
    mine = torch.tensor(splits, dtype=torch.int64, device=dev)
    theirs = torch.empty_like(mine)
    dist.all_to_all_single(theirs, mine, group=group)
    recv_splits = [int(v) for v in theirs.tolist()]
    rows = ep.be.empty_rows(sum(recv_splits), send)
    dist.all_to_all_single(rows, send, recv_splits, splits, group=group)
    expert = torch.empty(sum(recv_splits), dtype=send_expert.dtype, device=dev)
    dist.all_to_all_single(expert, send_expert, recv_splits, splits, group=group)
    y = ep.compute(rows, expert)
    back = ep.be.empty_rows(sum(splits), y)
    dist.all_to_all_single(back, y, splits, recv_splits, group=group)
    out = ep.finish(back)
    counts = ep.counts.clone()
    dist.all_reduce(counts, group=group)        # exact: integers
    return out, counts
