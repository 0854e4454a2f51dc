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

The exchange overlaps the computation: each rank's matrices are split into
``rounds`` groups of about equal cost, and after the local step of round g
every rank issues the (asynchronous) broadcasts of round g, which run while
round g + 1 is computed. All ranks derive the same rounds from the shape
table, so they issue the same collectives in the same order.
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


def assign_rounds(shapes: Sequence[Sequence[int]], owners: Sequence[int], world: int, rounds: int,
                  ns_steps: int = 5) -> List[List[List[int]]]:
    """rounds_of[r][g]: the matrices rank r updates in round g.

    Each rank's matrices, in index order, are cut into ``rounds`` consecutive
    groups by cumulative cost (a matrix goes to the round its cost midpoint
    falls in), so every round carries about 1/rounds of the rank's work.
    """
    if rounds < 1:
        raise ValueError("rounds must be >= 1")
    out = [[[] for _ in range(rounds)] for _ in range(world)]
    for r in range(world):
        mine = [i for i in range(len(shapes)) if owners[i] == r]
        costs = [step_cost(int(shapes[i][0]), int(shapes[i][1]), ns_steps) for i in mine]
        total = sum(costs)
        before = 0.0
        for i, c in zip(mine, costs):
            g = min(rounds - 1, int((before + 0.5 * c) * rounds / total)) if total > 0 else 0
            out[r][g].append(i)
            before += c
    return out


class LayerwiseMuon:
    """Muon over a process group with whole-matrix ownership.

    ``opt`` is a ``Muon`` handle on this rank's GPU (or any object whose
    ``step(params, grads, momenta, **kw)`` updates in place and skips
    ``None`` gradients). ``local_step`` overrides ``opt.step``.
    """

    def __init__(self, opt=None, group=None, local_step: Optional[Callable] = None, rounds: int = 4):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.opt = opt
        self.local_step = local_step if local_step is not None else opt.step
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        # One round when there is nothing to overlap with.
        self.rounds = 1 if self.world == 1 else int(rounds)
        self._owners = None
        self._rounds = None
        self._key = None

    def owners(self, shapes, ns_steps: int = 5) -> List[int]:
        key = (tuple(tuple(int(v) for v in s[:2]) for s in shapes), ns_steps)
        if key != self._key:
            self._owners = assign_owners(shapes, self.world, ns_steps)
            self._rounds = assign_rounds(shapes, self._owners, self.world, self.rounds, ns_steps)
            self._key = key
        return self._owners

    def step(self, params, grads, momenta, ns_steps: int = 5, **kw):
        """Update the matrices this rank owns, round by round, broadcasting
        each round's matrices from their owners while the next round runs.
        Every rank must call this with the same shapes."""
        shapes = [tuple(p.shape) for p in params]
        owners = self.owners(shapes, ns_steps)
        pending = []
        for g in range(self.rounds):
            mine = set(self._rounds[self.rank][g])
            if mine:
                local_grads = [gr if i in mine else None for i, gr in enumerate(grads)]
                self.local_step(params, local_grads, momenta, ns_steps=ns_steps, **kw)
            for i in sorted(i for r in range(self.world) for i in self._rounds[r][g]):
                src = owners[i] if self.group is None else self.dist.get_global_rank(self.group, owners[i])
                pending.append(self.dist.broadcast(params[i], src=src, group=self.group, async_op=True))
        for w in pending:
            w.wait()
        return owners
