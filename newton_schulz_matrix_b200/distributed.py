"""Sharded Muon step across ranks: one process per GPU, cost-balanced matrix
ownership, owner-only momentum, and an exchange of the updated weights.

Every matrix's orthogonalisation is independent, so the step shards by whole
matrices (the distributed orthogonalisation that the Moonlight catalogue note
attributes to the Moonlight work; the Gram Newton-Schulz write-up times a
pipeline-parallel share of Kimi K2).  Ownership is assigned longest-first to the
least-loaded rank (LPT) by the matrices' Newton-Schulz FLOPs.  Each rank runs
the library's fused step on the matrices it owns (momentum buffers live only
on the owner, as in a ZeRO-style sharded optimizer state) and then every
updated weight is broadcast from its owner, so all ranks end the step with the
full updated parameter set.  The caller provides each owner with its
gradients (e.g. after a reduce-scatter), as in any sharded optimizer.

The collective is torch.distributed's broadcast (NCCL over NVLink/NVSwitch on
GPUs); nothing here reads another GPU's memory directly.
"""
from __future__ import annotations

from typing import Callable, Sequence

import torch


def lpt_owners(costs: Sequence[float], world: int) -> list[int]:
    """Longest-processing-time assignment: visit items by decreasing cost (ties
    by index) and give each to the currently least-loaded rank (ties to the
    lowest rank).  Deterministic, so every rank computes the same plan."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(costs)), key=lambda i: (-float(costs[i]), i))
    load = [0.0] * world
    owner = [0] * len(costs)
    for i in order:
        r = min(range(world), key=lambda k: (load[k], k))
        owner[i] = r
        load[r] += float(costs[i])
    return owner


def ns_cost(shape, mode: str = "standard", iters: int = 5) -> float:
    """Newton-Schulz FLOPs of one matrix (the balancing weight)."""
    n, m = min(shape), max(shape)
    if mode == "standard":
        return iters * (4.0 * m * n * n + 2.0 * n ** 3)
    return 4.0 * m * n * n + (8.0 * iters) * n ** 3  # Gram forms: rectangular ends + n^3 chain


class ShardedMuonStep:
    """One Muon step over `params` sharded across the ranks of `group`.

    params  every rank's full list of weights (updated in place on all ranks)
    grads   gradients; only the entries this rank owns are read
    moms    momentum buffers for the owned entries: dict index -> fp32 tensor
    local_step_factory(params, grads, moms, **hp) -> callable running the local
            step; defaults to the library's fused MuonStep (CUDA)
    """

    def __init__(self, params: Sequence[torch.Tensor], grads: Sequence[torch.Tensor], moms: dict,
                 group=None, local_step_factory: Callable | None = None, **hp):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.params = list(params)
        mode = hp.get("mode", "standard")
        iters = len(hp.get("coeffs", ((0, 0, 0),) * 5))
        self.owner = lpt_owners([ns_cost(p.shape, mode, iters) for p in self.params], self.world)
        self.mine = [i for i, r in enumerate(self.owner) if r == self.rank]
        missing = [i for i in self.mine if i not in moms]
        if missing:
            raise ValueError(f"rank {self.rank} owns matrices {missing[:8]} but has no momentum buffer for them")
        if local_step_factory is None:
            from . import MuonStep as local_step_factory  # noqa: N813
        self.local = None
        if self.mine:
            self.local = local_step_factory([self.params[i] for i in self.mine], [grads[i] for i in self.mine],
                                            [moms[i] for i in self.mine], **hp)

    def owned(self) -> list[int]:
        return list(self.mine)

    def __call__(self) -> None:
        if self.local is not None:
            self.local()
        # every rank takes the same collective steps in the same order
        works = []
        for i, p in enumerate(self.params):
            src = self.dist.get_global_rank(self.group, self.owner[i]) if self.group is not None else self.owner[i]
            works.append(self.dist.broadcast(p, src=src, group=self.group, async_op=True))
        for w in works:
            w.wait()
