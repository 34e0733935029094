"""Sharding the scoring pass over ranks (one process per GPU).

Layers are independent, so each rank scores a subset of them; the only exchange is the
per-layer score vector (a few hundred floats), gathered so that every rank can run the
same deterministic selection.  Layers go to ranks by longest-processing-time-first on
their element counts, which keeps the per-rank byte counts within one layer of each
other.  The partition is a pure function of the layer sizes, so every rank knows every
other rank's layers without exchanging them.
"""
from typing import List, Sequence

import torch
import torch.distributed as dist


def lpt_partition(sizes: Sequence[int], world: int) -> List[List[int]]:
    """Layer indices per rank: largest layers first, each to the least-loaded rank (ties to
    the lower rank).  Every rank's list is returned in ascending layer order."""
    if world < 1:
        raise ValueError("world size must be >= 1")
    load = [0] * world
    parts: List[List[int]] = [[] for _ in range(world)]
    for i in sorted(range(len(sizes)), key=lambda j: (-sizes[j], j)):
        r = min(range(world), key=lambda q: (load[q], q))
        parts[r].append(i)
        load[r] += sizes[i]
    return [sorted(p) for p in parts]


class ScoreGather:
    """All-gather of per-rank score slices into the full [num_layers] vector.

    Built once per partition; ``__call__`` issues one all_gather on the current stream
    and one scatter, with no host synchronisation, so it can sit inside a timed loop."""

    def __init__(self, parts: List[List[int]], rank: int, num_layers: int, device, group=None):
        self.parts, self.rank, self.group = parts, rank, group
        self.width = max(1, max(len(p) for p in parts))
        idx = torch.full((len(parts), self.width), num_layers, dtype=torch.int64)
        for r, p in enumerate(parts):
            idx[r, : len(p)] = torch.as_tensor(p, dtype=torch.int64)
        self.index = idx.reshape(-1).to(device)  # padding points at a spare slot
        self.num_layers = num_layers
        self.n_local = len(parts[rank])

    def __call__(self, local_scores: torch.Tensor) -> torch.Tensor:
        dev, dt = local_scores.device, local_scores.dtype
        send = torch.zeros(self.width, dtype=dt, device=dev)
        send[: self.n_local] = local_scores[: self.n_local]
        recv = torch.empty(len(self.parts) * self.width, dtype=dt, device=dev)
        dist.all_gather_into_tensor(recv, send, group=self.group)
        out = torch.zeros(self.num_layers + 1, dtype=dt, device=dev)
        out.index_copy_(0, self.index, recv)
        return out[: self.num_layers]
