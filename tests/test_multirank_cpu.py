"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

With N GPUs every rank runs its own full matrix set (weak scaling, no
collective on the data path); the only collective is the max over ranks of
the step time, and the reference arm runs on rank 0 alone.
"""

import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(torch, dist, 10.0 * (rank + 1), torch.device("cpu"))
        # An error on one rank is seen by all (every rank takes the same branch).
        ok_all = bench.all_ranks_ok(torch, dist, torch.device("cpu"), True)
        ok_one_bad = bench.all_ranks_ok(torch, dist, torch.device("cpu"), rank != 1)
        out[rank] = (got, ok_all, ok_one_bad)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    world = 2
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0] == (20.0, True, False) and out[1] == (20.0, True, False)


def test_max_over_ranks_single_process():
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(torch, dist, 3.5, torch.device("cpu")) == 3.5
    assert bench.all_ranks_ok(torch, dist, torch.device("cpu"), False) is False


def test_reference_arm_non_zero_rank_exits_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_prints_one_json_line():
    import json
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        env.pop(k, None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "single", "--steps", "2", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "steps/s" and d["value"] > 0
    assert d["higher_is_better"] is True and d["steps"] == 2 and d["warmup"] == 3
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
