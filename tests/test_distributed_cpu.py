"""Layer-wise distributed Muon on CPU ranks (gloo, world size 2 and 3).

Every rank holds the same data-parallel state; each updates only the whole
matrices it owns (the local step here is the float64 oracle, standing in for
the GPU step on these CPU ranks) and every matrix is then broadcast from its
owner: all ranks must end with the parameters of a single-process step, and
each momentum is updated on its owner only.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from muon_newton_schulz_03_b200.distributed import assign_owners, assign_rounds, step_cost

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SHAPES = [(64, 96), (96, 64), (32, 32), (128, 40), (40, 128), (16, 200), (48, 48)]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    rng = np.random.default_rng(40)
    ps = [rng.standard_normal(s) * 0.02 for s in SHAPES]
    gs = [rng.standard_normal(s) for s in SHAPES]
    ms = [rng.standard_normal(s) * 0.01 for s in SHAPES]
    return ps, gs, ms


def _oracle_step(params, grads, momenta, ns_steps=5, **kw):
    import sys
    sys.path.insert(0, ROOT)
    from oracle import muon_oracle as O
    for p, g, m in zip(params, grads, momenta):
        if g is None:
            continue
        p2, m2, _, _ = O.muon_step_matrix(p.numpy(), g.numpy(), m.numpy(), ns_steps=ns_steps, **kw)
        p.copy_(torch.from_numpy(p2))
        m.copy_(torch.from_numpy(m2))


def _worker(rank, world, port, out, rounds=4):
    import torch.distributed as dist
    from muon_newton_schulz_03_b200.distributed import LayerwiseMuon
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ps, gs, ms = _inputs()
        P = [torch.tensor(p) for p in ps]
        G = [torch.tensor(g) for g in gs]
        M = [torch.tensor(m) for m in ms]
        lw = LayerwiseMuon(group=None, local_step=_oracle_step, rounds=rounds)
        owners = lw.step(P, G, M, lr=0.01, beta=0.9, wd=0.1)
        out[rank] = ([p.numpy() for p in P], [m.numpy() for m in M], owners)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,rounds", [(2, 1), (2, 4), (3, 2), (3, 9)])
def test_layerwise_step_matches_single_process(world, rounds):
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, port, out, rounds), nprocs=world, join=True)
    ps, gs, ms = _inputs()
    P = [torch.tensor(p) for p in ps]
    M = [torch.tensor(m) for m in ms]
    _oracle_step(P, [torch.tensor(g) for g in gs], M, lr=0.01, beta=0.9, wd=0.1)
    owners = out[0][2]
    assert sorted(set(owners)) == list(range(world))
    for r in range(world):
        got_p, got_m, own = out[r]
        assert own == owners
        for i in range(len(SHAPES)):
            assert np.array_equal(got_p[i], P[i].numpy())          # broadcast from the owner
            if owners[i] == r:
                assert np.array_equal(got_m[i], M[i].numpy())      # momentum updated by its owner
            else:
                assert np.array_equal(got_m[i], ms[i])             # untouched elsewhere


def test_assignment_is_balanced_and_deterministic():
    import workloads as W
    shapes = W.llama3_8b_shapes()
    for world in (1, 2, 4, 8):
        owners = assign_owners(shapes, world)
        assert owners == assign_owners(shapes, world)
        load = [0.0] * world
        for (m, n), r in zip(shapes, owners):
            load[r] += step_cost(m, n)
        # greedy LPT: the spread is at most one matrix's cost
        assert max(load) - min(load) <= max(step_cost(m, n) for m, n in shapes) + 1e-12
    assert assign_owners([(8, 8)], 4) == [0]
    with pytest.raises(ValueError):
        assign_owners(shapes, 0)


def test_rounds_cover_each_owned_matrix_once():
    import workloads as W
    shapes = W.llama3_8b_shapes()
    for world in (2, 4, 8):
        owners = assign_owners(shapes, world)
        for rounds in (1, 3, 4, 16):
            rr = assign_rounds(shapes, owners, world, rounds)
            assert rr == assign_rounds(shapes, owners, world, rounds)
            for r in range(world):
                flat = [i for g in rr[r] for i in g]
                assert sorted(flat) == [i for i in range(len(shapes)) if owners[i] == r]
                assert flat == sorted(flat)                     # consecutive, index order
                costs = [sum(step_cost(*shapes[i]) for i in g) for g in rr[r]]
                biggest = max(step_cost(*shapes[i]) for i in flat)
                share = sum(costs) / rounds
                assert all(abs(c - share) <= biggest for c in costs)   # within one matrix of even
    with pytest.raises(ValueError):
        assign_rounds(shapes, assign_owners(shapes, 2), 2, 0)
