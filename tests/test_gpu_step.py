"""GPU parity of the whole Muon step (muon_step through the C ABI).

* the single 256 x 512 workload and the GPT-2-small set in full;
* the Llama-3-8B and MoE sets at full size in the launch configuration the
  benchmark times, checked on sampled matrices that the oracle recomputes;
* edge cases: skipped matrices, zero gradients, zero iterations, NaNs,
  repeated steps (momentum carried), CUDA-graph replay, status word.
"""

import numpy as np
import pytest
import torch

import muon_newton_schulz_03_b200 as muon
import workloads as W
from oracle import muon_oracle as O

from gpu_helpers import (DEV, TOL_BF16_NS, TOL_ELEM, TOL_FP32_NS, bf16_ns_tolerance, bf16_program_error, cuda_bf16,
                         cuda_f32, gate_bf16_update, make_set, rel, report, to64, workspace_matrix, x_buffer)

pytestmark = pytest.mark.gpu

F32 = lambda v: float(np.float32(v))  # noqa: E731  (scalars as the kernels see them)


def _step_fused(opt, shapes, active=None):
    """Whether a step of `opt` on these shapes writes p' in its last combine
    and stores no O (muon_config.fused_apply): the handle allows it, and no
    active matrix is on the small path or has rows whose length is not a
    multiple of four."""
    if not opt.fused_apply:
        return False
    small = set(muon.plan_query(shapes, opt.ns_precision, opt.small_path, opt.cta_pair)["small"])
    idx = range(len(shapes)) if active is None else active
    return not any(i in small for i in idx) and all(shapes[i][1] % 4 == 0 for i in idx)


def _check_step(cpu, dev, shapes, opt, *, lr, beta, wd, nesterov=True, ns_steps=5, scale_mode=O.SCALE_MOONLIGHT,
                tol=TOL_BF16_NS, check_o=True, indices=None, gram_mats=(), coeffs=O.DEFAULT_COEFFS, tag=""):
    """Every checked matrix against the exact oracle: momentum at 1e-6; O and
    the update at the bf16 gate (bf16 mode: 2e-2, or the pages' own bf16
    program's frozen distance where that is larger; ``tol`` for zero
    iterations) or at ``tol`` (fp32 debug mode); p' at 1e-6 with the oracle
    fed the GPU's own O. A handle whose last iteration writes p' itself
    (``fused_apply``) leaves no O in the workspace: there the update alone is
    checked (its gate carries O's tolerance)."""
    indices = range(len(shapes)) if indices is None else indices
    worst = 0.0
    bf16 = opt.ns_precision == "bf16"
    for i in indices:
        m, n = shapes[i]
        p0, g, m0 = cpu[i]
        p_ref, m_ref, o_ref, nu = O.muon_step_matrix(p0, g, m0, lr=F32(lr), beta=F32(beta), nesterov=nesterov,
                                                     wd=F32(wd), ns_steps=ns_steps, coeffs=coeffs,
                                                     scale_mode=scale_mode)
        p_gpu, _, m_gpu = (to64(t) for t in dev[i])
        assert rel(m_gpu, m_ref) <= TOL_ELEM, f"momentum of matrix {i}"
        scale = O.update_scale(m, n, scale_mode)
        if bf16 and ns_steps > 0:
            u = O.nesterov_blend(g, m_ref, F32(beta), nesterov)
            tol_o = bf16_ns_tolerance(u, ns_steps, coeffs)
        else:
            tol_o = tol
        e = gate_bf16_update(p_gpu, p0, p_ref, o_ref, F32(lr) * scale, tol_o, f"{tag} matrix {i} {m}x{n}")
        worst = max(worst, e)
        if check_o and ns_steps > 0 and not _step_fused(opt, shapes, indices):
            dtype = torch.bfloat16 if bf16 else torch.float32
            flips = (ns_steps + 1) // 2 if gram_mats else ns_steps
            o_gpu = to64(workspace_matrix(opt, shapes, i, flips % 2, dtype)[:, :n])
            eo = rel(o_gpu, o_ref)
            report(f"O {tag} matrix {i} {m}x{n}", eo, tol_o,
                   bf16_program_error(u, ns_steps, coeffs) if bf16 and ns_steps > 0 else None)
            assert eo <= tol_o, f"matrix {i} {m}x{n}: O off by {eo:.3e} (gate {tol_o:.3e})"
            # p' itself at the elementwise gate, with the oracle fed the GPU's O.
            p_from_o = O.apply_update(p0, o_gpu, F32(lr), F32(wd), scale)
            assert rel(p_gpu, p_from_o) <= TOL_ELEM
    return worst


@pytest.mark.parametrize("prec,tol", [("bf16", TOL_BF16_NS), ("fp32", TOL_FP32_NS)])
def test_single_matrix_workload(prec, tol):
    # One 256 x 512 fp32 gradient, zero momentum, beta 0.95 Nesterov, 5 steps,
    # lr 0.02, wd 0, Jordan scale (the lr 0.02 pairing).
    shapes = W.single_shapes()
    cpu, dev = make_set(W.CONFIG_SINGLE, shapes, torch.float32)
    # O stored (fused_apply off), so that it is checked as well as p'.
    opt = muon.Muon(device=0, scale_mode="jordan", ns_precision=prec, fused_apply=False)
    opt.step([d[0] for d in dev], [d[1] for d in dev], [d[2] for d in dev], lr=0.02, beta=0.95, wd=0.0)
    torch.cuda.synchronize()
    _check_step(cpu, dev, shapes, opt, lr=0.02, beta=0.95, wd=0.0, scale_mode=O.SCALE_JORDAN, tol=tol,
                tag=f"config single {prec}")
    assert opt.status() == (0, 0, 0)
    assert opt.last_launch_count() == (17 if prec == "bf16" else 1 + 15 + 1)
    opt.close()


@pytest.mark.parametrize("prec,tol,pair", [("bf16", TOL_BF16_NS, True), ("bf16", TOL_BF16_NS, False),
                                           ("fp32", TOL_FP32_NS, True)])
def test_gpt2_small_set(prec, tol, pair):
    shapes = W.gpt2_shapes()
    cpu, dev = make_set(W.CONFIG_GPT2, shapes, torch.float32)
    opt = muon.Muon(device=0, ns_precision=prec, cta_pair=pair, fused_apply=False)   # O stored and checked
    opt.step([d[0] for d in dev], [d[1] for d in dev], [d[2] for d in dev], lr=2e-4, beta=0.95, wd=0.1)
    torch.cuda.synchronize()
    idx = range(len(shapes)) if prec == "bf16" else range(4)
    _check_step(cpu, dev, shapes, opt, lr=2e-4, beta=0.95, wd=0.1, tol=tol, indices=idx,
                tag=f"config gpt2 {prec} {'pair' if pair else 'single'}")
    assert opt.status() == (0, 0, 0)
    opt.close()


def test_warm_momentum_three_steps():
    # Three consecutive steps with fresh gradients: the momentum carried on
    # the GPU matches the oracle's recurrence.
    shapes = [(256, 768), (768, 256)]
    opt = muon.Muon(device=0)
    rng = np.random.default_rng(20)
    p = [cuda_f32(rng.standard_normal(s) * 0.02) for s in shapes]
    mo = [torch.zeros(s, dtype=torch.float32, device=DEV) for s in shapes]
    p64 = [to64(t) for t in p]
    p_start = [x.copy() for x in p64]
    m64 = [np.zeros(s) for s in shapes]
    for step in range(3):
        g = [cuda_f32(W.gradient_cpu(W.CONFIG_GPT2, m, n, 100 + 10 * step + i)) for i, (m, n) in enumerate(shapes)]
        opt.step(p, g, mo, lr=2e-4, beta=0.95, wd=0.1)
        for i in range(len(shapes)):
            p64[i], m64[i], _, _ = O.muon_step_matrix(p64[i], to64(g[i]), m64[i], lr=F32(2e-4), beta=F32(0.95),
                                                      wd=F32(0.1))
    torch.cuda.synchronize()
    for i in range(len(shapes)):
        assert rel(to64(mo[i]), m64[i]) <= 1e-6
        # total displacement over the three steps (well-conditioned inputs:
        # bf16 arithmetic meets the exact gate here)
        assert rel(to64(p[i]) - p_start[i], p64[i] - p_start[i]) <= TOL_BF16_NS
    opt.close()


def test_skipped_zero_and_nan_gradients():
    shapes = [(64, 96), (96, 64), (32, 32), (48, 80)]
    opt = muon.Muon(device=0, check_nonfinite=True)
    rng = np.random.default_rng(21)
    p = [cuda_f32(rng.standard_normal(s)) for s in shapes]
    mo = [cuda_f32(rng.standard_normal(s) * 0.1) for s in shapes]
    p0 = [to64(t) for t in p]
    m0 = [to64(t) for t in mo]
    g = [None, torch.zeros(shapes[1], dtype=torch.float32, device=DEV),
         cuda_f32(rng.standard_normal(shapes[2])), cuda_f32(rng.standard_normal(shapes[3]))]
    opt.step(p, g, mo, lr=0.01, beta=0.9, wd=0.5, nesterov=False)
    torch.cuda.synchronize()
    # Skipped: untouched.
    assert np.array_equal(to64(p[0]), p0[0]) and np.array_equal(to64(mo[0]), m0[0])
    # Zero gradient with non-zero momentum and Nesterov off: u = 0.9 m; a
    # plain Muon step of that direction.
    kw = dict(lr=F32(0.01), beta=F32(0.9), wd=F32(0.5), nesterov=False)
    ref, mref, oref, _ = O.muon_step_matrix(p0[1], np.zeros(shapes[1]), m0[1], **kw)
    u = O.nesterov_blend(np.zeros(shapes[1]), mref, F32(0.9), False)
    gate_bf16_update(to64(p[1]), p0[1], ref, oref, F32(0.01) * O.update_scale(96, 64), bf16_ns_tolerance(u),
                     "zero-gradient matrix")
    assert opt.status() == (0, 0, 0)
    # A NaN is counted and reported.
    g[2][3, 4] = float("nan")
    g[3][0, 0] = float("inf")
    opt.step(p, g, mo, lr=0.01, beta=0.9, wd=0.5)
    code, ew, nf = opt.status()
    assert code == 5 and ew == 0 and nf == 2
    assert opt.status() == (0, 0, 0)  # cleared
    opt.close()


def test_truly_zero_state_gives_pure_decay():
    shapes = [(40, 60)]
    opt = muon.Muon(device=0)
    p = [cuda_f32(np.random.default_rng(22).standard_normal(shapes[0]))]
    p0 = to64(p[0])
    opt.step(p, [torch.zeros(shapes[0], device=DEV)], [torch.zeros(shapes[0], device=DEV)], lr=0.1, wd=0.2)
    torch.cuda.synchronize()
    assert rel(to64(p[0]), p0 * (1 - F32(0.1) * F32(0.2))) <= TOL_ELEM
    opt.close()


def test_zero_iterations():
    shapes = [(30, 50), (50, 30)]
    cpu, dev = make_set(W.CONFIG_GPT2, shapes, torch.float32)
    opt = muon.Muon(device=0)
    opt.step([d[0] for d in dev], [d[1] for d in dev], [d[2] for d in dev], lr=0.01, ns_steps=0)
    torch.cuda.synchronize()
    _check_step(cpu, dev, shapes, opt, lr=0.01, beta=0.95, wd=0.1, ns_steps=0, tol=4e-3, check_o=False)
    opt.close()


def test_repeat_runs_agree_and_graph_replay():
    shapes = W.gpt2_shapes()[:8]
    cpu, dev = make_set(W.CONFIG_GPT2, shapes, torch.float32)
    base_p = [d[0].clone() for d in dev]
    outs = []
    opt = muon.Muon(device=0)
    for _ in range(2):
        p = [t.clone() for t in base_p]
        mo = [torch.zeros_like(t) for t in base_p]
        opt.step(p, [d[1] for d in dev], mo, lr=2e-4)
        torch.cuda.synchronize()
        outs.append([to64(t) for t in p])
    for a, b in zip(*outs):
        assert np.max(np.abs(a - b)) <= 1e-9
    # Capture the same call (same pointers: no table upload) in a CUDA graph.
    p = [t.clone() for t in base_p]
    mo = [torch.zeros_like(t) for t in base_p]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        opt.step(p, [d[1] for d in dev], mo, lr=2e-4)       # warm: plan and tables exist
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    for t, b in zip(p, base_p):
        t.copy_(b)
    for t in mo:
        t.zero_()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        opt.step(p, [d[1] for d in dev], mo, lr=2e-4)
    for t, b in zip(p, base_p):
        t.copy_(b)
    for t in mo:
        t.zero_()
    graph.replay()
    torch.cuda.synchronize()
    for a, b in zip(outs[0], p):
        assert np.max(np.abs(a - to64(b))) <= 1e-9
    opt.close()


@pytest.mark.parametrize("shapes", [
    [(128, 384), (384, 128), (100, 100)],
    # more chunks than staging slots (slots are reused), mixed paths, one
    # matrix without a gradient
    [(256, 768), (768, 256), (64, 64), (1024, 512), (300, 700), (512, 1024), (128, 128), (640, 320),
     (256, 256), (200, 600), (900, 300), (384, 384)],
    # no small-path matrix: the last combine of each chunk writes p' into
    # the staging slot through the parameter maps of the staging pointers
    [(256, 768), (768, 256), (1024, 512), (512, 1024), (300, 700), (700, 300)],
])
def test_step_host_matches_device_step(shapes):
    cpu, dev = make_set(W.CONFIG_GPT2, shapes, torch.bfloat16)
    hp = [d[0].cpu().pin_memory() for d in dev]
    hg = [d[1].cpu().pin_memory() for d in dev]
    hm = [d[2].cpu().pin_memory() for d in dev]
    p0 = [t.clone() for t in hp]
    skip = 5 if len(shapes) > 5 else None
    if skip is not None:
        hg[skip] = None
    opt = muon.Muon(device=0)
    opt.step_host(hp, hg, hm, lr=2e-4)
    torch.cuda.synchronize()
    dg = [None if g is None else d[1] for g, d in zip(hg, dev)]
    opt.step([d[0] for d in dev], dg, [d[2] for d in dev], lr=2e-4)
    torch.cuda.synchronize()
    for i in range(len(shapes)):
        ref_p, ref_m = dev[i][0].cpu(), dev[i][2].cpu()
        if i == skip:
            assert torch.equal(hp[i], p0[i])
        assert torch.equal(hm[i], ref_m)
        # The norm's double-precision atomics may round in a different order:
        # allow a few float32 ulps.
        assert torch.max(torch.abs(hp[i] - ref_p)) <= 1e-6 * (torch.max(torch.abs(ref_p)) + 1e-30)
    assert opt.status() == (0, 0, 0)
    opt.close()


def test_bounded_wait_expiry_reports_timeout_and_recovers():
    # A wait limit far below any real wait makes the first pending wait run
    # out: the kernel records the error word, drains its copies and MMAs,
    # frees tensor memory and returns. The context stays usable.
    shapes = W.PARITY_SHAPES["wait"]
    cpu, dev = make_set(W.CONFIG_GPT2, shapes, torch.float32)
    opt = muon.Muon(device=0, wait_timeout_s=1e-9)
    opt.step([d[0].clone() for d in dev], [d[1] for d in dev], [d[2].clone() for d in dev], lr=2e-4)
    code, ew, nf = opt.status()
    assert code == 4 and ew in (1, 2, 3, 4)
    opt.close()
    ok = muon.Muon(device=0)
    ok.step([d[0] for d in dev], [d[1] for d in dev], [d[2] for d in dev], lr=2e-4)
    torch.cuda.synchronize()
    _check_step(cpu, dev, shapes, ok, lr=2e-4, beta=0.95, wd=0.1)
    assert ok.status() == (0, 0, 0)
    ok.close()


def test_invalid_arguments_rejected():
    opt = muon.Muon(device=0)
    p = torch.zeros((8, 8), device=DEV)
    with pytest.raises(muon.MuonError) as e:
        opt.step([p], [p], [p], lr=0.1)        # overlapping buffers
    assert e.value.code == 1
    with pytest.raises(muon.MuonError):
        opt.step([p], [torch.zeros((8, 8), device=DEV)], [torch.zeros((8, 8), device=DEV)], lr=0.1, beta=1.5)
    with pytest.raises(muon.MuonError):
        opt.step([p], [torch.zeros((8, 8), device=DEV)], [torch.zeros((8, 8), device=DEV)], lr=0.1, ns_steps=65)
    big = torch.zeros(64, device=DEV)
    with pytest.raises(muon.MuonError):   # misaligned pointer
        opt.step([big[1:].view(7, 9)], [torch.zeros((7, 9), device=DEV)], [torch.zeros((7, 9), device=DEV)], lr=0.1)
    opt.close()


# ---------------------------------------------------------------------------
# Full-size sets in the benchmark's launch configuration, sampled matrices
# ---------------------------------------------------------------------------

def _full_set_sampled(config, shapes, grad_dtype, sample, lr=2e-4, wd=0.1, tag=""):
    dev = []
    cpu = W.set_values(config, shapes, grad_dtype == torch.bfloat16, indices=sample)
    for i, (m, n) in enumerate(shapes):
        seed = W.seed_for(config, i // 7, i % 7)
        if i in sample:
            p, g, _ = cpu[i]
            gt = cuda_bf16(g) if grad_dtype == torch.bfloat16 else cuda_f32(g)
            pt = cuda_f32(p)
            assert np.array_equal(to64(gt), g) and np.array_equal(to64(pt), p)
        else:
            gt = W.gradient_gpu(config, m, n, seed, DEV, grad_dtype)
            pt = W.param_gpu(m, n, seed, DEV)
        dev.append((pt, gt, torch.zeros((m, n), dtype=torch.float32, device=DEV)))
    opt = muon.Muon(device=0)
    opt.step([d[0] for d in dev], [d[1] for d in dev], [d[2] for d in dev], lr=lr, beta=0.95, wd=wd)
    torch.cuda.synchronize()
    assert opt.status() == (0, 0, 0)
    errs = []
    for i in sample:
        m, n = shapes[i]
        p0, g, m0 = cpu[i]
        kw = dict(lr=F32(lr), beta=F32(0.95), wd=F32(wd))
        p_ref, m_ref, o_ref, _ = O.muon_step_matrix(p0, g, m0, **kw)
        p_gpu, m_gpu = to64(dev[i][0]), to64(dev[i][2])
        assert rel(m_gpu, m_ref) <= TOL_ELEM
        u = O.nesterov_blend(g, m_ref, F32(0.95))
        tol_o = bf16_ns_tolerance(u)
        errs.append((gate_bf16_update(p_gpu, p0, p_ref, o_ref, F32(lr) * O.update_scale(m, n), tol_o,
                                      f"config {tag} matrix {i} {m}x{n}"), tol_o))
    # The bench's configuration: the last iteration writes p' itself, so the
    # update's gate (which carries O's tolerance) is the check; no O is stored.
    assert opt.fused_apply and opt.last_launch_count() == 1 + 15
    opt.close()
    return errs


@pytest.mark.slow
def test_llama3_8b_set_sampled():
    shapes = W.llama3_8b_shapes()
    # layer 0 q (square), k (wide, small), gate (tall), and layer 31 down (wide)
    _full_set_sampled(W.CONFIG_LLAMA, shapes, torch.bfloat16, sample=W.LLAMA_SAMPLE, tag="llama3")


@pytest.mark.slow
def test_moe_set_sampled():
    shapes = W.moe_shapes()
    # three experts: gate (wide) and down (tall). Condition number 1e4: the
    # pages' own bf16 program lands above 2e-2 here, and the gate is its
    # frozen distance from exact.
    _full_set_sampled(W.CONFIG_MOE, shapes, torch.bfloat16, sample=W.MOE_SAMPLE, tag="moe")


def test_mixed_small_and_tiled_matrices_in_one_step():
    # Matrices on the on-chip path and on the tiled phases in the same call:
    # both land in the same workspace buffer before the apply kernel.
    shapes = W.PARITY_SHAPES["mixed"]
    plan = muon.plan_query(shapes)
    assert plan["small"] == [0, 1, 2, 4, 6]
    cpu, dev = make_set(W.CONFIG_GPT2, shapes, torch.float32)
    opt = muon.Muon(device=0)
    opt.step([d[0] for d in dev], [d[1] for d in dev], [d[2] for d in dev], lr=2e-4, beta=0.95, wd=0.1)
    torch.cuda.synchronize()
    _check_step(cpu, dev, shapes, opt, lr=2e-4, beta=0.95, wd=0.1)
    assert opt.last_launch_count() == 1 + 1 + 15 + 1   # K1, small path, phases, apply (a small matrix)
    assert opt.status() == (0, 0, 0)
    opt.close()


@pytest.mark.parametrize("ns_steps", [5, 4, 1])
def test_gram_form_step(ns_steps):
    # The Gram form on the tiled phases: wide, tall, square and ragged
    # matrices, one-step and two-step segments. The small path (kept in the
    # standard form) handles the small matrices of the same call.
    shapes = W.PARITY_SHAPES["gram"]
    plan = muon.plan_query(shapes)
    cpu, dev = make_set(W.CONFIG_GPT2, shapes, torch.float32)
    opt = muon.Muon(device=0, ns_algorithm="gram")
    opt.step([d[0] for d in dev], [d[1] for d in dev], [d[2] for d in dev], lr=2e-4, beta=0.95, wd=0.1,
             ns_steps=ns_steps)
    torch.cuda.synchronize()
    tiled = [i for i in range(len(shapes)) if i not in plan["small"]]
    _check_step(cpu, dev, shapes, opt, lr=2e-4, beta=0.95, wd=0.1, ns_steps=ns_steps, gram_mats=tiled)
    segs2, segs1 = ns_steps // 2, ns_steps % 2
    assert opt.last_launch_count() == 1 + 1 + 7 * segs2 + 3 * segs1 + 1
    assert opt.status() == (0, 0, 0)
    opt.close()


FUSED_CASES = {
    "single": (W.CONFIG_SINGLE, W.single_shapes(), torch.float32, None),
    "gpt2": (W.CONFIG_GPT2, W.gpt2_shapes()[:8], torch.bfloat16, None),
    # ragged edges: the bulk copies of p clip rows and columns past the matrix
    "ragged": (W.CONFIG_GPT2, [(300, 700), (1000, 200), (520, 520), (768, 2304), (2304, 768), (200, 1000)],
               torch.float32, None),
    "split": (W.CONFIG_GPT2, W.PARITY_SHAPES["split"], torch.float32, W.SPLIT_ROWS),
    # not fused (a small-path matrix; rows whose length is not a multiple of 4)
    "mixed": (W.CONFIG_GPT2, W.PARITY_SHAPES["mixed"], torch.float32, None),
    "odd_rows": (W.CONFIG_GPT2, [(300, 701), (1000, 201)], torch.float32, None),
}


@pytest.mark.parametrize("case", sorted(FUSED_CASES))
def test_fused_apply_is_bitwise_the_separate_pass(case):
    # Where a step qualifies, its last combine writes p' = p (1 - lr wd) -
    # lr scale O itself (O rounded to bf16 first; p moved by bulk copies):
    # p' and m' are bitwise those of the separate apply pass on the same
    # inputs (fixed-order norm), with one launch fewer. Where it does not, the
    # separate pass runs in both handles.
    config, shapes, gdtype, splits = FUSED_CASES[case]
    cpu, dev = make_set(config, shapes, gdtype)
    twin = [(p.clone(), g.clone(), m.clone()) for (p, g, m) in dev]
    fused = muon.Muon(device=0, deterministic=True)
    separate = muon.Muon(device=0, deterministic=True, fused_apply=False)
    kw = dict(lr=2e-4, beta=0.95, wd=0.1, row_splits=splits)
    fused.step([d[0] for d in dev], [d[1] for d in dev], [d[2] for d in dev], **kw)
    separate.step([t[0] for t in twin], [t[1] for t in twin], [t[2] for t in twin], **kw)
    torch.cuda.synchronize()
    for i, ((p, _, m), (p2, _, m2)) in enumerate(zip(dev, twin)):
        assert torch.equal(m, m2), f"momentum of matrix {i}"
        assert torch.equal(p, p2), f"p' of matrix {i}: {float(torch.max(torch.abs(p - p2))):.3e} apart"
    expect_fused = case not in ("mixed", "odd_rows")
    assert separate.last_launch_count() == fused.last_launch_count() + (1 if expect_fused else 0)
    assert fused.status() == (0, 0, 0) and separate.status() == (0, 0, 0)
    fused.close()
    separate.close()


def test_deterministic_norm_is_bitwise_repeatable():
    # Fixed-order norm sums: two steps on identical copies of the inputs give
    # identical bits, and the step still meets the oracle's gates.
    shapes = W.PARITY_SHAPES["deterministic"]
    cpu, dev = make_set(W.CONFIG_GPT2, shapes, torch.float32)
    twin = [(p.clone(), g.clone(), m.clone()) for (p, g, m) in dev]
    opt = muon.Muon(device=0, deterministic=True)
    for d in (dev, twin):
        opt.step([x[0] for x in d], [x[1] for x in d], [x[2] for x in d], lr=2e-4, beta=0.95, wd=0.1)
    torch.cuda.synchronize()
    for (p, _, m), (p2, _, m2) in zip(dev, twin):
        assert torch.equal(p, p2) and torch.equal(m, m2)
    _check_step(cpu, dev, shapes, opt, lr=2e-4, beta=0.95, wd=0.1)
    assert opt.last_launch_count() == 1 + 1 + 1 + 15 + 1   # K1, fixed-order sum, small path, phases, apply
    # The stage entry point: the same sums as the atomic mode to fp64 rounding.
    ref = muon.Muon(device=0)
    sums = []
    for o in (opt, ref):
        moms = [torch.zeros(s, dtype=torch.float32, device=DEV) for s in shapes]
        ys = [x_buffer(m, n) for (m, n) in shapes]
        ss = torch.zeros(len(shapes), dtype=torch.float64, device=DEV)
        o.momentum_norm([x[1] for x in twin], moms, ys, ss, beta=0.95)
        sums.append(ss.cpu().numpy())
    torch.cuda.synchronize()
    assert opt.last_launch_count() == 2
    assert np.allclose(sums[0], sums[1], rtol=1e-13, atol=0)
    assert opt.status() == (0, 0, 0)
    opt.close()
    ref.close()


def test_gram_form_rejected_with_fp32_or_pairs():
    for kw in (dict(ns_precision="fp32"), dict(cta_pair=True)):
        with pytest.raises(muon.MuonError):
            muon.Muon(device=0, ns_algorithm="gram", **kw)


def test_split_muon_qkv_and_per_head():
    # QKV fused weight cut into Q, K, V; an attention output projection cut
    # per head (12 heads of 64 rows); one matrix kept whole.
    shapes = W.PARITY_SHAPES["split"]
    splits = W.SPLIT_ROWS
    cpu, dev = make_set(W.CONFIG_GPT2, shapes, torch.float32)
    opt = muon.Muon(device=0)
    opt.step([d[0] for d in dev], [d[1] for d in dev], [d[2] for d in dev], lr=2e-4, wd=0.1, row_splits=splits)
    torch.cuda.synchronize()
    assert opt.status() == (0, 0, 0)
    assert opt.last_launch_count() >= 16
    for i, (m, n) in enumerate(shapes):
        p0, g, m0 = cpu[i]
        rows = m if splits[i] is None else splits[i]
        kw = dict(lr=F32(2e-4), beta=F32(0.95), wd=F32(0.1))
        p_ref, m_ref, o_ref, _ = O.muon_step_matrix_split(p0, g, m0, [rows] * (m // rows), **kw)
        assert rel(to64(dev[i][2]), m_ref) <= TOL_ELEM
        p_gpu = to64(dev[i][0])
        for r0 in range(0, m, rows):
            sl = slice(r0, r0 + rows)
            u = O.nesterov_blend(g[sl], m_ref[sl], F32(0.95))
            gate_bf16_update(p_gpu[sl], p0[sl], p_ref[sl], o_ref[sl], F32(2e-4) * O.update_scale(rows, n),
                             bf16_ns_tolerance(u), f"split matrix {i} rows {r0}..{r0 + rows}")
    opt.close()


def test_coefficient_schedule():
    shapes = W.PARITY_SHAPES["schedule"]
    cpu, dev = make_set(W.CONFIG_GPT2, shapes, torch.float32)
    base = [(d[0].clone(), d[2].clone()) for d in dev]
    opt = muon.Muon(device=0)
    # A constant table is the plain step, bit for bit.
    opt.step_schedule([d[0] for d in dev], [d[1] for d in dev], [d[2] for d in dev], [O.DEFAULT_COEFFS] * 5, lr=2e-4)
    torch.cuda.synchronize()
    p_sched = [to64(d[0]) for d in dev]
    for d, (p0, m0) in zip(dev, base):
        d[0].copy_(p0)
        d[2].copy_(m0)
    opt.step([d[0] for d in dev], [d[1] for d in dev], [d[2] for d in dev], lr=2e-4)
    torch.cuda.synchronize()
    for a, d in zip(p_sched, dev):
        assert np.max(np.abs(a - to64(d[0]))) <= 1e-6 * np.max(np.abs(a))
    # A varying table against the oracle.
    table = W.SCHEDULE_TABLE
    for d, (p0, m0) in zip(dev, base):
        d[0].copy_(p0)
        d[2].copy_(m0)
    opt.step_schedule([d[0] for d in dev], [d[1] for d in dev], [d[2] for d in dev], table, lr=2e-4)
    torch.cuda.synchronize()
    _check_step(cpu, dev, shapes, opt, lr=2e-4, beta=0.95, wd=0.1, ns_steps=4, check_o=False,
                coeffs=[tuple(F32(v) for v in r) for r in table])
    with pytest.raises(ValueError):
        opt.step_schedule([d[0] for d in dev], [d[1] for d in dev], [d[2] for d in dev], [], lr=2e-4)
    assert opt.status() == (0, 0, 0)
    opt.close()


def test_qk_clip_matches_oracle():
    rng = np.random.default_rng(31)
    heads, d, dm = 8, 64, 512
    wq = cuda_f32(rng.standard_normal((heads * d, dm)) * 0.02)
    wk = cuda_f32(rng.standard_normal((heads // 2 * d, dm)) * 0.02)       # grouped K heads
    sq = torch.tensor([250.0, 30.0, 101.0, 100.0, float("nan"), 5000.0, -3.0, 99.9], dtype=torch.float32,
                      device=DEV)
    sk = torch.tensor([250.0, 101.0, 5000.0, 99.9], dtype=torch.float32, device=DEV)
    q0, k0 = to64(wq), to64(wk)
    opt = muon.Muon(device=0)
    opt.qk_clip([wq, wk], [sq, sk], [d, d], tau=100.0)
    torch.cuda.synchronize()
    assert rel(to64(wq), O.qk_clip(q0, sq.cpu().numpy(), 100.0, d)) <= TOL_ELEM
    assert rel(to64(wk), O.qk_clip(k0, sk.cpu().numpy(), 100.0, d)) <= TOL_ELEM
    assert np.array_equal(to64(wq)[64:128], q0[64:128])          # 30 < tau: untouched
    opt.close()


def test_layerwise_single_rank_matches_oracle():
    # The layer-wise distributed wrapper over an NCCL group of one rank:
    # every matrix is owned locally, computed in cost-balanced rounds, and
    # broadcast to self. Checked against the oracle like the plain step.
    import socket
    import torch.distributed as dist
    from muon_newton_schulz_03_b200.distributed import LayerwiseMuon
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        shapes = W.PARITY_SHAPES["layerwise"]
        cpu, dev = make_set(W.CONFIG_GPT2, shapes, torch.float32)
        opt = muon.Muon(device=0)
        LayerwiseMuon(opt).step([d[0] for d in dev], [d[1] for d in dev], [d[2] for d in dev], lr=2e-4)
        torch.cuda.synchronize()
        assert opt.status() == (0, 0, 0)
        _check_step(cpu, dev, shapes, opt, lr=2e-4, beta=0.95, wd=0.1, check_o=False)
        opt.close()
    finally:
        dist.destroy_process_group()


def _group_launches(plan, bounds, deterministic=True, fused=False):
    """Launches of a grouped step: per group K1 (+ fixed-order sum), the
    small path if the group has small matrices, 15 phases if it has tiled
    ones, and the apply kernel unless the last phases write p' themselves."""
    small = set(plan["small"])
    total = 0
    for g0, g1 in zip(bounds[:-1], bounds[1:]):
        mats = range(g0, g1)
        total += 1 + (0 if fused else 1) + (1 if deterministic else 0)
        total += 1 if any(i in small for i in mats) else 0
        total += 15 if any(i not in small for i in mats) else 0
    return total


def test_workspace_cap_runs_groups_and_matches_uncapped():
    # A cap of a third of the workspace packs the matrices into groups that
    # share one workspace and run one after another. In the fixed-order norm
    # mode the result is bitwise the uncapped step's (every tile computes the
    # same products), and it meets the oracle's gates; the stage call and
    # the host-buffer step run the same groups.
    shapes = W.PARITY_SHAPES["layerwise"]
    full = muon.plan_query(shapes)["ws_bytes"]
    cap = full // 3
    bounds = muon.plan_groups(shapes, cap)["bounds"]
    assert len(bounds) - 1 >= 3
    cpu, dev = make_set(W.CONFIG_GPT2, shapes, torch.float32)
    twin = [(p.clone(), g.clone(), m.clone()) for (p, g, m) in dev]
    capped = muon.Muon(device=0, workspace_cap_bytes=cap, deterministic=True)
    plain = muon.Muon(device=0, deterministic=True)
    capped.step([d[0] for d in dev], [d[1] for d in dev], [d[2] for d in dev], lr=2e-4, beta=0.95, wd=0.1)
    plain.step([t[0] for t in twin], [t[1] for t in twin], [t[2] for t in twin], lr=2e-4, beta=0.95, wd=0.1)
    torch.cuda.synchronize()
    assert capped.workspace()[1] <= cap
    assert capped.last_launch_count() == _group_launches(muon.plan_query(shapes), bounds)
    for (p, _, m), (p2, _, m2) in zip(dev, twin):
        assert torch.equal(p, p2) and torch.equal(m, m2)
    _check_step(cpu, dev, shapes, capped, lr=2e-4, beta=0.95, wd=0.1, check_o=False)
    assert capped.status() == (0, 0, 0)
    # The stage call under the cap.
    xin = [x_buffer(m, n, fill=W.gaussian_set([(m, n)], 50 + i)[0]) for i, (m, n) in enumerate(shapes)]
    sumsq = torch.tensor([float(torch.sum(x[:, :n].double() ** 2)) for x, (m, n) in zip(xin, shapes)],
                         dtype=torch.float64, device=DEV)
    outs = [[x_buffer(m, n) for (m, n) in shapes] for _ in range(2)]
    capped.newton_schulz(xin, outs[0], shapes, sumsq, ns_steps=5)
    plain.newton_schulz(xin, outs[1], shapes, sumsq, ns_steps=5)
    torch.cuda.synchronize()
    for a, b, (m, n) in zip(outs[0], outs[1], shapes):
        assert torch.equal(a[:, :n], b[:, :n])
    # The host-buffer step under the cap: the same groups, bitwise the device step.
    hp = [t[0].cpu().pin_memory() for t in twin]
    hg = [t[1].cpu().pin_memory() for t in twin]
    hm = [t[2].cpu().pin_memory() for t in twin]
    capped.step_host(hp, hg, hm, lr=2e-4)
    capped.step([d[0] for d in dev], [d[1] for d in dev], [d[2] for d in dev], lr=2e-4)
    torch.cuda.synchronize()
    for a, d in zip(hp, dev):
        assert torch.equal(a, d[0].cpu())
    assert capped.status() == (0, 0, 0)
    capped.close()
    plain.close()
    tight = muon.Muon(device=0, workspace_cap_bytes=1 << 20)
    with pytest.raises(muon.MuonError) as e:    # a matrix above the cap on its own
        tight.step([d[0] for d in dev], [d[1] for d in dev], [d[2] for d in dev], lr=2e-4)
    assert e.value.code == 3
    tight.close()


def test_workspace_cap_with_the_update_in_the_last_combine():
    # Groups under a workspace cap on a set without small-path matrices: each
    # group's last combine writes p' (no apply launch), bitwise the uncapped
    # step's in the fixed-order norm mode (whose update is gated against the
    # oracle by the other step tests).
    shapes = [(256, 768), (768, 256), (1024, 512), (512, 1024), (300, 700), (700, 300)]
    cap = muon.plan_query(shapes)["ws_bytes"] // 3
    bounds = muon.plan_groups(shapes, cap)["bounds"]
    assert len(bounds) - 1 >= 3
    cpu, dev = make_set(W.CONFIG_GPT2, shapes, torch.float32)
    twin = [(p.clone(), g.clone(), m.clone()) for (p, g, m) in dev]
    capped = muon.Muon(device=0, workspace_cap_bytes=cap, deterministic=True)
    plain = muon.Muon(device=0, deterministic=True)
    capped.step([d[0] for d in dev], [d[1] for d in dev], [d[2] for d in dev], lr=2e-4, beta=0.95, wd=0.1)
    plain.step([t[0] for t in twin], [t[1] for t in twin], [t[2] for t in twin], lr=2e-4, beta=0.95, wd=0.1)
    torch.cuda.synchronize()
    assert _step_fused(capped, shapes)
    assert capped.last_launch_count() == _group_launches(muon.plan_query(shapes), bounds, fused=True)
    for (p, _, m), (p2, _, m2) in zip(dev, twin):
        assert torch.equal(p, p2) and torch.equal(m, m2)
    assert capped.status() == (0, 0, 0) and plain.status() == (0, 0, 0)
    capped.close()
    plain.close()


def test_fresh_pointers_every_step_match_fixed_pointers():
    # A training loop that hands over new gradient and momentum tensors each
    # step (a fresh allocation per step): the pointer tables go through the
    # handle's ring of device slots with stream-ordered uploads, more steps
    # than slots. The parameters and momenta match the fixed-pointer run
    # bitwise (fixed-order norm), and the step time stays close to it.
    shapes = W.gpt2_shapes()[:8] + [(64, 64), (300, 700)]
    steps = 20
    grads = [[cuda_f32(W.gradient_cpu(W.CONFIG_GPT2, m, n, 900 + 31 * k + i)) for i, (m, n) in enumerate(shapes)]
             for k in range(4)]
    p0 = [cuda_f32(W.param_cpu(m, n, i)) for i, (m, n) in enumerate(shapes)]
    opt = muon.Muon(device=0, deterministic=True)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]

    def run(fresh):
        p = [t.clone() for t in p0]
        mo = [torch.zeros_like(t) for t in p0]
        g = [torch.empty_like(t) for t in p0]
        total = 0.0
        for k in range(steps):
            if fresh:
                g = [t.clone() for t in grads[k % 4]]
                mo = [t.clone() for t in mo]
            else:
                for dst, src in zip(g, grads[k % 4]):
                    dst.copy_(src)
            ev[0].record()
            opt.step(p, g, mo, lr=2e-4)
            ev[1].record()
            torch.cuda.synchronize()
            if k >= 2:
                total += ev[0].elapsed_time(ev[1])
        return p, mo, total

    p_fix, m_fix, t_fix = run(False)
    p_new, m_new, t_new = run(True)
    for a, b in zip(p_fix, p_new):
        assert torch.equal(a, b)
    for a, b in zip(m_fix, m_new):
        assert torch.equal(a, b)
    assert opt.status() == (0, 0, 0)
    print(f"fixed pointers {t_fix / (steps - 2):.3f} ms/step, fresh pointers {t_new / (steps - 2):.3f} ms/step")
    assert t_new <= 1.25 * t_fix + 0.05 * (steps - 2)
    opt.close()


def test_steps_over_a_subset_launch_only_its_tiles():
    # Matrices without a gradient drop out of the tile lists: a step over a
    # subset (one round of layer-wise Muon) launches over the active
    # matrices' tiles only, and matches the oracle on them while the others
    # stay untouched.
    shapes = W.PARITY_SHAPES["layerwise"]
    cpu, dev = make_set(W.CONFIG_GPT2, shapes, torch.float32)
    before = [(d[0].clone(), d[2].clone()) for d in dev]
    opt = muon.Muon(device=0)
    opt.profile_enable(1)
    active = {1, 4}                 # two tiled matrices
    g = [d[1] if i in active else None for i, d in enumerate(dev)]
    opt.step([d[0] for d in dev], g, [d[2] for d in dev], lr=2e-4)
    torch.cuda.synchronize()
    prof = opt.profile_read()
    opt.profile_enable(0)
    kinds = [k for k, _ in prof]
    assert kinds.count("ns_gram") == kinds.count("ns_poly") == kinds.count("ns_comb") == 5
    assert "ns_small" not in kinds          # the small matrix (64 x 64) has no gradient
    for i, d in enumerate(dev):
        if i not in active:
            assert torch.equal(d[0], before[i][0]) and torch.equal(d[2], before[i][1])
    _check_step(cpu, dev, shapes, opt, lr=2e-4, beta=0.95, wd=0.1, indices=sorted(active))
    assert opt.status() == (0, 0, 0)
    opt.close()


def test_captured_graph_keeps_its_tables_while_pointers_churn():
    # A step captured in a CUDA graph keeps pointing at the device tables of
    # its pointer set: those ring slots are pinned, so ten uncaptured steps
    # with fresh tensors (more than the ring's eight slots) do not overwrite
    # them, and a replay afterwards still updates the captured tensors exactly
    # as an uncaptured step does. A new pointer set during capture is refused.
    shapes = W.gpt2_shapes()[:4]
    cpu, dev = make_set(W.CONFIG_GPT2, shapes, torch.float32)
    base_p = [d[0].clone() for d in dev]
    opt = muon.Muon(device=0, deterministic=True)
    p = [t.clone() for t in base_p]
    mo = [torch.zeros_like(t) for t in base_p]
    g = [d[1] for d in dev]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        opt.step(p, g, mo, lr=2e-4)                      # tables for these pointers exist
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        opt.step(p, g, mo, lr=2e-4)
    # Churn: ten steps on fresh tensors each time.
    for k in range(10):
        fp = [t.clone() for t in base_p]
        fm = [torch.zeros_like(t) for t in base_p]
        fg = [t.clone() for t in g]
        opt.step(fp, fg, fm, lr=2e-4)
    torch.cuda.synchronize()
    want_p = [t.clone() for t in base_p]
    want_m = [torch.zeros_like(t) for t in base_p]
    opt.step(want_p, g, want_m, lr=2e-4)
    for t, b in zip(p, base_p):
        t.copy_(b)
    for t in mo:
        t.zero_()
    graph.replay()
    torch.cuda.synchronize()
    for a, b in zip(p, want_p):
        assert torch.equal(a, b)
    for a, b in zip(mo, want_m):
        assert torch.equal(a, b)
    # New pointers while capturing: refused (the upload cannot be captured).
    other = [t.clone() for t in base_p]
    s2 = torch.cuda.Stream()
    s2.wait_stream(torch.cuda.current_stream())
    g2 = torch.cuda.CUDAGraph()
    with pytest.raises(muon.MuonError):
        with torch.cuda.graph(g2, stream=s2):
            opt.step(other, g, [torch.zeros_like(t) for t in base_p], lr=2e-4)
    del graph
    assert opt.status() == (0, 0, 0)
    opt.close()
