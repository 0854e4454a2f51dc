"""Auxiliary checks on the GPU: workspace canaries and checkpoint / resume.

* Canary bytes written over the whole workspace survive a step wherever the
  plan puts no data: no kernel writes outside its regions (the sum-of-squares
  block and each matrix's X0, X1, A, B).
* The library keeps no optimizer state besides the caller's parameters and
  momenta: two steps, a save to host memory, a fresh handle, a reload and two
  more steps give the same bits as four uninterrupted steps (with the
  fixed-order norm sums).
"""

import numpy as np
import pytest
import torch

import muon_newton_schulz_03_b200 as muon
import workloads as W

from gpu_helpers import DEV, _CudaArray, make_set

pytestmark = pytest.mark.gpu

CANARY = 0xA5


def _byte_view(ptr, nbytes):
    torch.cuda.synchronize()
    return torch.as_tensor(_CudaArray(ptr, (nbytes,), "|u1"), device=DEV)


def test_workspace_outside_regions_keeps_its_canary():
    shapes = [(1, 1), (7, 3), (127, 129), (300, 100), (64, 1000), (1000, 64), (513, 257), (128, 512)]
    cpu, dev = make_set(W.CONFIG_GPT2, shapes, torch.float32)
    opt = muon.Muon(device=0)
    args = ([d[0] for d in dev], [d[1] for d in dev], [d[2] for d in dev])
    opt.step(*args, lr=2e-4)                        # plan and workspace exist
    base, size = opt.workspace()
    ws = _byte_view(base, size)
    ws.fill_(CANARY)
    opt.step(*args, lr=2e-4)
    torch.cuda.synchronize()
    plan = muon.plan_query(shapes)
    used = torch.zeros(size, dtype=torch.bool, device=DEV)
    used[:8 * len(shapes)] = True                  # per-matrix sums of squares
    for (m, n), offs in zip(shapes, plan["region_offsets"]):
        s = min(m, n)
        lens = [m * muon.round_up(n, 8) * 2] * 2 + [s * muon.round_up(s, 8) * 2] * 2
        for o, ln in zip(offs, lens):
            used[o:o + ln] = True
    outside = ws[~used]
    assert outside.numel() > 0
    assert bool((outside == CANARY).all()), f"{int((outside != CANARY).sum())} bytes outside the regions changed"
    # and the step itself still ran: every region holds written data somewhere
    assert bool((ws[used] != CANARY).any())
    assert opt.status() == (0, 0, 0)
    opt.close()


def test_checkpoint_resume_is_bitwise():
    shapes = [(256, 768), (768, 256), (300, 1000), (64, 96)]
    rng = np.random.default_rng(77)
    p0 = [rng.standard_normal(s).astype(np.float32) * 0.02 for s in shapes]
    grads = [[torch.tensor(rng.standard_normal(s).astype(np.float32), device=DEV) for s in shapes]
             for _ in range(4)]

    def run(steps, p, m, opt):
        for k in steps:
            opt.step(p, grads[k], m, lr=2e-4, beta=0.95, wd=0.1)
        torch.cuda.synchronize()

    # four uninterrupted steps
    opt = muon.Muon(device=0, deterministic=True)
    pa = [torch.tensor(x, device=DEV) for x in p0]
    ma = [torch.zeros(s, dtype=torch.float32, device=DEV) for s in shapes]
    run(range(4), pa, ma, opt)
    opt.close()

    # two steps, checkpoint to host, a fresh handle, reload, two more steps
    opt = muon.Muon(device=0, deterministic=True)
    pb = [torch.tensor(x, device=DEV) for x in p0]
    mb = [torch.zeros(s, dtype=torch.float32, device=DEV) for s in shapes]
    run(range(2), pb, mb, opt)
    saved = ([t.cpu().clone() for t in pb], [t.cpu().clone() for t in mb])
    opt.close()
    del pb, mb
    opt = muon.Muon(device=0, deterministic=True)
    pc = [t.to(DEV) for t in saved[0]]
    mc = [t.to(DEV) for t in saved[1]]
    run(range(2, 4), pc, mc, opt)
    for x, y in zip(pa + ma, pc + mc):
        assert torch.equal(x, y)
    assert opt.status() == (0, 0, 0)
    opt.close()
