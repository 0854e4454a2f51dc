"""Layer-wise distributed Muon: whole matrices owned by data-parallel ranks.

"Why Muon Works", section 7 (and 7.2): tag the 2D hidden matrices, assign
each whole matrix (or structured block) to one DP rank, let every rank run
the Muon update only for the matrices it owns, then all-gather / sync the
parameters so the next forward sees the same weights everywhere. The Muon
state (momentum) of a matrix lives on its owner only.

Here the owner's update is the library's ordinary step with the gradients of
other ranks' matrices passed as ``None`` (skipped: their parameters and
momenta are left untouched); the exchange is one broadcast per matrix from
its owner over the process group (NCCL over NVLink on GPUs, gloo on CPU).
Ownership is a longest-processing-time packing of the matrices by their
estimated step time, so ranks finish their local steps together.
"""

from __future__ import annotations

from typing import Callable, List, Optional, Sequence

# Rates used only to weigh matrices against each other when packing.
_TENSOR_FLOPS = 1.4e15      # sustained bf16 tensor rate, FLOP/s
_HBM_BYTES = 6.5e12         # HBM bandwidth, B/s


def step_cost(m: int, n: int, ns_steps: int = 5, grad_bytes: int = 4) -> float:
    """Estimated seconds of one Muon step on an m x n matrix: nominal
    Newton-Schulz FLOPs on the tensor cores plus the elementwise bytes."""
    s, l = min(m, n), max(m, n)
    flops = ns_steps * (4.0 * s * s * l + 2.0 * s ** 3)
    nbytes = m * n * (grad_bytes + 4 + 4 + 2 + 4 + 2 + 4)
    return flops / _TENSOR_FLOPS + nbytes / _HBM_BYTES


def assign_owners(shapes: Sequence[Sequence[int]], world: int, ns_steps: int = 5) -> List[int]:
    """Owner rank of every matrix: greedy longest-processing-time packing.

    Matrices are taken by decreasing cost (ties by index) and each goes to
    the rank with the smallest load so far (ties by rank). Deterministic, so
    every rank computes the same assignment from the same shape table.
    """
    if world < 1:
        raise ValueError("world size must be >= 1")
    costs = [step_cost(int(s[0]), int(s[1]), ns_steps) for s in shapes]
    order = sorted(range(len(shapes)), key=lambda i: (-costs[i], i))
    load = [0.0] * world
    owners = [0] * len(shapes)
    for i in order:
        r = min(range(world), key=lambda k: (load[k], k))
        owners[i] = r
        load[r] += costs[i]
    return owners


class LayerwiseMuon:
    """Muon over a process group with whole-matrix ownership.

    ``opt`` is a ``Muon`` handle on this rank's GPU (or any object whose
    ``step(params, grads, momenta, **kw)`` updates in place and skips
    ``None`` gradients). ``local_step`` overrides ``opt.step``.
    """

    def __init__(self, opt=None, group=None, local_step: Optional[Callable] = None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.opt = opt
        self.local_step = local_step if local_step is not None else opt.step
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self._owners = None
        self._key = None

    def owners(self, shapes, ns_steps: int = 5) -> List[int]:
        key = (tuple(tuple(int(v) for v in s[:2]) for s in shapes), ns_steps)
        if key != self._key:
            self._owners = assign_owners(shapes, self.world, ns_steps)
            self._key = key
        return self._owners

    def step(self, params, grads, momenta, ns_steps: int = 5, **kw):
        """Update the matrices this rank owns, then broadcast every matrix
        from its owner. Every rank must call this with the same shapes."""
        shapes = [tuple(p.shape) for p in params]
        owners = self.owners(shapes, ns_steps)
        local_grads = [g if owners[i] == self.rank else None for i, g in enumerate(grads)]
        if any(g is not None for g in local_grads):
            self.local_step(params, local_grads, momenta, ns_steps=ns_steps, **kw)
        for i, p in enumerate(params):
            src = owners[i] if self.group is None else self.dist.get_global_rank(self.group, owners[i])
            self.dist.broadcast(p, src=src, group=self.group)
        return owners
