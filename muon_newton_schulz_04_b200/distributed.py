"""Matrix-sharded Muon over data-parallel ranks (one process per GPU).

Every matrix's step is independent ("Muon: An optimizer for hidden layers in
neural networks", section 4 defines the update per matrix), so under data
parallelism -- every rank holds the same, already averaged gradients -- rank r
steps only the matrices it owns and keeps only their momentum buffers (the
optimizer-state sharding of the Moonlight result's Distributed Muon, whole
matrices instead of row slices, so no gradient needs gathering).  One collective
then hands every rank the updated weights: each rank packs its updated matrices
into one flat buffer, and a single all-gather (NCCL over NVLink on GPUs, gloo in
the CPU tests) delivers all shards.

Ownership is decided once by longest-processing-time-first on the nominal
Newton-Schulz FLOPs 5 (4 m^2 n + 2 m^3) of each matrix, so ranks finish at about
the same time.  All Muon arithmetic runs in the CUDA library; this module only
partitions, packs and calls the collective.
"""
from __future__ import annotations

import heapq
from typing import Callable, List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist


def ns_flops(rows: int, cols: int, ns_steps: int = 5) -> float:
    m, n = min(rows, cols), max(rows, cols)
    return ns_steps * (4.0 * m * m * n + 2.0 * m ** 3)


def lpt_partition(costs: Sequence[float], world: int) -> List[List[int]]:
    """Greedy longest-processing-time assignment: items in decreasing cost, each to
    the currently least-loaded rank (ties to the lower rank).  Returns the item
    indices of each rank in increasing order."""
    if world < 1:
        raise ValueError("world must be >= 1")
    heap = [(0.0, r) for r in range(world)]
    parts: List[List[int]] = [[] for _ in range(world)]
    for i in sorted(range(len(costs)), key=lambda k: (-costs[k], k)):
        load, r = heapq.heappop(heap)
        parts[r].append(i)
        heapq.heappush(heap, (load + costs[i], r))
    return [sorted(p) for p in parts]


class ShardedMuon:
    """Muon over a list of 2D weights, sharded by whole matrices across ranks.

    shapes: (rows, cols) of every matrix, identical on all ranks.
    local_step(W_own, G_own, B_own): runs the Muon step of the rank's own matrices
    in place (by default the CUDA library's muon_step through the binding).
    """

    def __init__(self, shapes: Sequence[Tuple[int, int]], cfg=None, group=None, device=None,
                 local_step: Optional[Callable] = None):
        self.shapes = [tuple(s) for s in shapes]
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        steps = getattr(cfg, "ns_steps", 5) if cfg is not None else 5
        self.parts = lpt_partition([ns_flops(r, c, steps) for (r, c) in self.shapes], self.world)
        self.own = self.parts[self.rank]
        self.shard_elems = [sum(self.shapes[k][0] * self.shapes[k][1] for k in p) for p in self.parts]
        self.max_elems = max(self.shard_elems) if self.shard_elems else 0
        if local_step is None:
            from . import Group, Muon
            opt = Muon(cfg, device=0 if device is None else device)

            def local_step(W, G, B):
                groups = {}
                for w, g, b in zip(W, G, B):
                    groups.setdefault(tuple(w.shape), []).append((w, g, b))
                opt.step([Group(W=[x[0] for x in v], G=[x[1] for x in v], B=[x[2] for x in v])
                          for v in groups.values()])
            self._opt = opt
        self.local_step = local_step

    def new_momentum(self, like: Sequence[torch.Tensor]) -> List[torch.Tensor]:
        """Zeroed fp32 momentum buffers for the rank's own matrices only."""
        return [torch.zeros_like(like[k], dtype=torch.float32) for k in self.own]

    def step(self, W: Sequence[torch.Tensor], G: Sequence[torch.Tensor], B_own: Sequence[torch.Tensor]) -> None:
        """One step: update the own matrices, then all-gather every shard into W."""
        self.local_step([W[k] for k in self.own], [G[k] for k in self.own], list(B_own))
        if self.world == 1:
            return
        dev = W[0].device
        send = torch.zeros(self.max_elems, dtype=W[0].dtype, device=dev)
        off = 0
        for k in self.own:
            n = W[k].numel()
            send[off:off + n].copy_(W[k].reshape(-1))
            off += n
        recv = torch.empty(self.world * self.max_elems, dtype=W[0].dtype, device=dev)
        dist.all_gather_into_tensor(recv, send, group=self.group)
        for r, part in enumerate(self.parts):
            if r == self.rank:
                continue
            off = r * self.max_elems
            for k in part:
                n = W[k].numel()
                W[k].copy_(recv[off:off + n].view_as(W[k]))
                off += n
