"""The compute steps of mixture_experts_layer_28_b200.ep on the host, from
the fp64 oracle: a test backend for the expert-parallel orchestration on CPU
process groups (gloo).  TEST INFRASTRUCTURE: the library never uses it."""
from __future__ import annotations

import numpy as np
import torch

from oracle import moe_zc_ref as ref


class OracleBackend:
    def route(self, x, router, N, Z, K):
        r = ref.route(x, router.W_r, router.b, N, K, router.logit_offset)
        idx = torch.from_numpy(r.idx.astype(np.int32))
        return (idx, torch.from_numpy(r.gate), torch.from_numpy(r.zsum),
                torch.from_numpy(ref.expert_load(r.idx, N + Z).astype(np.int32)))

    def dispatch(self, x, idx, counts, N, rows):
        """FFN picks packed by expert (expert 0 first), (token, pick) order
        inside an expert; slot -1 for zero-expert picks."""
        ix = idx.numpy()
        T, K = ix.shape
        slot = np.full((T, K), -1, dtype=np.int32)
        order = sorted((int(ix[t, k]), t, k) for t in range(T) for k in range(K) if ix[t, k] < N)
        assert len(order) == rows
        src = np.zeros(rows, dtype=np.int64)
        expert = np.zeros(rows, dtype=np.int32)
        for s, (e, t, k) in enumerate(order):
            slot[t, k] = s
            src[s] = t
            expert[s] = e
        xs = torch.from_numpy(ref._f64(x))
        return torch.from_numpy(slot), xs[torch.from_numpy(src)], torch.from_numpy(expert)

    def experts(self, rows, expert, shard):
        y = torch.zeros(rows.shape, dtype=torch.float64)
        ex = expert.numpy()
        for e in np.unique(ex):
            sel = np.nonzero(ex == e)[0]
            j = int(e) - shard.base
            y[sel] = torch.from_numpy(ref.swiglu_expert(rows[sel].numpy(), shard.W_gate[j],
                                                        shard.W_up[j], shard.W_down[j]))
        return y

    def combine(self, x, y_rows, slot, gate, zsum):
        xs = ref._f64(x)
        sl, g = slot.numpy(), gate.numpy()
        out = zsum.numpy()[:, None] * xs
        yr = y_rows.numpy()
        for t in range(xs.shape[0]):
            for k in range(sl.shape[1]):
                if sl[t, k] >= 0:
                    out[t] += g[t, k] * yr[sl[t, k]]
        return torch.from_numpy(out)

    def empty_rows(self, n, like):
        return torch.empty(n, *like.shape[1:], dtype=like.dtype)
