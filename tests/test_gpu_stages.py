"""GPU parity of each stage of the step against the float64 oracle.

Stage 1 (momentum, Nesterov, norm, cast), stage 2 (Newton-Schulz on the
tensor cores, and the fp32 debug path), stage 3 (apply), each called
through the C ABI on seeded inputs of several tile counts with ragged tails.
"""

import numpy as np
import pytest
import torch

import muon_newton_schulz_03_b200 as muon
from oracle import muon_oracle as O

from gpu_helpers import (DEV, TOL_BF16_NS, TOL_ELEM, TOL_FP32_NS, TOL_GPU_VS_GPU, bf16_ulp, cuda_bf16, gate_bf16_ns,
                         gaussian_buffers,
                         cuda_f32, rel, to64, x_buffer)

pytestmark = pytest.mark.gpu

import workloads as W  # noqa: E402

RAGGED = W.PARITY_SHAPES["ragged"]


@pytest.fixture(scope="module")
def opt_bf16():
    h = muon.Muon(device=0)
    yield h
    h.close()


@pytest.fixture(scope="module")
def opts():
    """Handles for both tiled-phase kernels: single CTAs (default) and CTA pairs."""
    hs = {"pair": muon.Muon(device=0, cta_pair=True), "single": muon.Muon(device=0)}
    yield hs
    for h in hs.values():
        h.close()


@pytest.fixture(scope="module")
def opt_fp32():
    h = muon.Muon(device=0, ns_precision="fp32")
    yield h
    h.close()


def _assert_status_clean(opt):
    code, ew, nf = opt.status()
    assert (code, ew, nf) == (0, 0, 0), f"device status {code} error word {ew} non-finite {nf}"


# ---------------------------------------------------------------------------
# Stage 1
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("grad_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("nesterov", [True, False])
def test_momentum_norm_matches_oracle(opt_bf16, grad_dtype, nesterov):
    rng = np.random.default_rng(1)
    shapes = RAGGED
    beta = np.float32(0.95)
    gs, ms, ys, gd, md = [], [], [], [], []
    for (m, n) in shapes:
        g = rng.standard_normal((m, n)) * 1e-2
        mom = rng.standard_normal((m, n)) * 1e-2
        gt = cuda_bf16(g) if grad_dtype == torch.bfloat16 else cuda_f32(g)
        mt = cuda_f32(mom)
        gs.append(to64(gt)); ms.append(to64(mt))
        gd.append(gt); md.append(mt); ys.append(x_buffer(m, n))
    # one skipped matrix
    gd[3] = None
    sumsq = torch.full((len(shapes),), -1.0, dtype=torch.float64, device=DEV)
    opt_bf16.momentum_norm(gd, md, ys, sumsq, beta=float(beta), nesterov=nesterov)
    torch.cuda.synchronize()
    ss = sumsq.cpu().numpy()
    for i, (m, n) in enumerate(shapes):
        if i == 3:
            assert np.array_equal(to64(md[i]), ms[i])
            assert ss[i] == 0.0
            continue
        m_ref = O.momentum_update(ms[i], gs[i], float(beta))
        u_ref = O.nesterov_blend(gs[i], m_ref, float(beta), nesterov)
        assert rel(to64(md[i]), m_ref) <= TOL_ELEM
        nu_ref = np.linalg.norm(u_ref)
        assert abs(np.sqrt(ss[i]) - nu_ref) <= TOL_ELEM * nu_ref
        y = to64(ys[i][:, :n])
        y_ref = O.bf16_round(u_ref)
        # One bf16 ulp, plus the float32 rounding of the lerp chain that
        # produces u on the GPU (it matters where u nearly cancels).
        fp32_err = 8 * 2.0 ** -24 * (np.abs(gs[i]) + np.abs(m_ref) + np.abs(ms[i]))
        bad = np.abs(y - y_ref) > bf16_ulp(y_ref) + fp32_err
        assert not bad.any(), f"matrix {i}: {bad.sum()} casts off by more than one bf16 ulp"


def test_momentum_norm_fp32_output(opt_fp32):
    rng = np.random.default_rng(2)
    shapes = [(33, 70), (128, 256), (7, 8)]
    gd = [cuda_f32(rng.standard_normal(s)) for s in shapes]
    md = [cuda_f32(rng.standard_normal(s)) for s in shapes]
    g64 = [to64(t) for t in gd]
    m64 = [to64(t) for t in md]
    ys = [x_buffer(m, n, torch.float32) for (m, n) in shapes]
    sumsq = torch.zeros(len(shapes), dtype=torch.float64, device=DEV)
    opt_fp32.momentum_norm(gd, md, ys, sumsq, beta=0.9, nesterov=True)
    torch.cuda.synchronize()
    for i, (m, n) in enumerate(shapes):
        m_ref = O.momentum_update(m64[i], g64[i], float(np.float32(0.9)))
        u_ref = O.nesterov_blend(g64[i], m_ref, float(np.float32(0.9)))
        assert rel(to64(ys[i][:, :n]), u_ref) <= TOL_ELEM
        assert rel(to64(md[i]), m_ref) <= TOL_ELEM


# ---------------------------------------------------------------------------
# Stage 3
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("mode", ["moonlight", "jordan", "bernstein", "none"])
def test_apply_matches_oracle(mode):
    opt = muon.Muon(device=0, scale_mode=mode, extra_scale=1.25)
    rng = np.random.default_rng(3)
    shapes = RAGGED
    pd, od, p64, o64 = [], [], [], []
    for (m, n) in shapes:
        pt = cuda_f32(rng.standard_normal((m, n)) * 0.02)
        ob = x_buffer(m, n, fill=rng.standard_normal((m, n)) * 0.05)
        pd.append(pt); od.append(ob); p64.append(to64(pt)); o64.append(to64(ob[:, :n]))
    od[2] = None
    lr, wd = np.float32(2e-4), np.float32(0.1)
    opt.apply(pd, od, lr=float(lr), wd=float(wd))
    torch.cuda.synchronize()
    for i, (m, n) in enumerate(shapes):
        got = to64(pd[i])
        if i == 2:
            assert np.array_equal(got, p64[i])
            continue
        scale = O.update_scale(m, n, O.__dict__["SCALE_" + mode.upper()], float(np.float32(1.25)))
        ref = O.apply_update(p64[i], o64[i], float(lr), float(wd), scale)
        assert rel(got, ref) <= TOL_ELEM, f"matrix {i} {m}x{n}"
    opt.close()


def test_apply_with_norm_scale(opt_bf16):
    rng = np.random.default_rng(4)
    shapes = [(40, 72), (72, 40)]
    pd = [cuda_f32(rng.standard_normal(s)) for s in shapes]
    p64 = [to64(t) for t in pd]
    ob = [x_buffer(m, n, fill=rng.standard_normal((m, n))) for (m, n) in shapes]
    ss = np.array([4.0, 0.25])
    sumsq = torch.tensor(ss, dtype=torch.float64, device=DEV)
    opt_bf16.apply(pd, ob, lr=0.01, wd=0.0, sumsq=sumsq)
    torch.cuda.synchronize()
    for i, (m, n) in enumerate(shapes):
        o = to64(ob[i][:, :n]) / (np.sqrt(ss[i]) + O.EPS)
        ref = O.apply_update(p64[i], o, float(np.float32(0.01)), 0.0, O.update_scale(m, n))
        assert rel(to64(pd[i]), ref) <= TOL_ELEM


# ---------------------------------------------------------------------------
# Stage 2: Newton-Schulz
# ---------------------------------------------------------------------------

def _ns_inputs(shapes, seed, scale=1.0):
    return gaussian_buffers(shapes, seed, scale)


@pytest.mark.parametrize("kind", ["pair", "single"])
def test_ns_identity_combine_is_exact(opts, kind):
    # (a, b, c) = (1, 0, 0): B = a I + 0 = I, so X1 = I X = X exactly.
    # Exercises every tile's combine epilogue addressing (direct, ragged
    # tails, tall) and the diagonal of the polynomial's tiles.
    opt_bf16 = opts[kind]
    shapes = RAGGED
    xin, x64 = _ns_inputs(shapes, 5)
    xout = [x_buffer(m, n) for (m, n) in shapes]
    opt_bf16.newton_schulz(xin, xout, shapes, None, ns_steps=1, coeffs=(1.0, 0.0, 0.0))
    torch.cuda.synchronize()
    for i, (m, n) in enumerate(shapes):
        assert np.array_equal(to64(xout[i][:, :n]), x64[i]), f"matrix {i} {m}x{n}"
    _assert_status_clean(opt_bf16)


@pytest.mark.parametrize("kind", ["pair", "single"])
@pytest.mark.parametrize("coeffs", [(0.0, 1.0, 0.0), (0.0, 0.0, 1.0), (0.5, -0.25, 0.125)])
def test_ns_single_step_phases(opts, kind, coeffs):
    opt_bf16 = opts[kind]
    # One step with chosen coefficients isolates the Gram (b), the polynomial
    # product (c) and the combine (a) against float64 products of the same
    # bf16 input; alpha = 1 (no norm).
    shapes = RAGGED
    xin, x64 = _ns_inputs(shapes, 6, scale=0.05)
    xout = [x_buffer(m, n) for (m, n) in shapes]
    opt_bf16.newton_schulz(xin, xout, shapes, None, ns_steps=1, coeffs=coeffs)
    torch.cuda.synchronize()
    for i, (m, n) in enumerate(shapes):
        ref = O.ns_only(x64[i], 1, coeffs)
        got = to64(xout[i][:, :n])
        gate_bf16_ns(got, ref, x64[i], 1, coeffs, normalised=False, what=f"matrix {i} {m}x{n}")
    _assert_status_clean(opt_bf16)


@pytest.mark.parametrize("kind", ["pair", "single"])
@pytest.mark.parametrize("steps", [1, 2, 5])
def test_ns_bf16_matches_oracle(opts, kind, steps):
    opt_bf16 = opts[kind]
    shapes = RAGGED
    xin, x64 = _ns_inputs(shapes, 7 + steps)
    sumsq = torch.tensor([np.sum(x ** 2) for x in x64], dtype=torch.float64, device=DEV)
    xout = [x_buffer(m, n) for (m, n) in shapes]
    opt_bf16.newton_schulz(xin, xout, shapes, sumsq, ns_steps=steps)
    torch.cuda.synchronize()
    for i, (m, n) in enumerate(shapes):
        ref = O.newton_schulz(x64[i], steps)
        got = to64(xout[i][:, :n])
        gate_bf16_ns(got, ref, x64[i], steps, what=f"matrix {i} {m}x{n}")
    # Inputs were not modified.
    for i, (m, n) in enumerate(shapes):
        assert np.array_equal(to64(xin[i][:, :n]), x64[i])
    _assert_status_clean(opt_bf16)


def test_polynomial_identity_form_matches_bulk_load_form():
    # A polynomial launch whose matrices all have s < 2048 takes b A on the
    # tensor cores (scaled identities); a launch that also holds a larger
    # matrix reads A in the epilogue instead. The same short matrices (the
    # ragged inputs of the five-step test) through both forms: each within
    # its oracle gate, and the two within fp32 summation order of each other.
    h = muon.Muon(device=0, small_path=False)
    shapes, big = RAGGED, [(2048, 2048)]
    xin, x64 = _ns_inputs(shapes + big, 12)
    sumsq = torch.tensor([np.sum(x ** 2) for x in x64], dtype=torch.float64, device=DEV)
    short = len(shapes)
    out_ident = [x_buffer(m, n) for (m, n) in shapes]
    out_bulk = [x_buffer(m, n) for (m, n) in shapes + big]
    h.newton_schulz(xin[:short], out_ident, shapes, sumsq[:short].contiguous(), ns_steps=5)
    h.newton_schulz(xin, out_bulk, shapes + big, sumsq, ns_steps=5)
    torch.cuda.synchronize()
    for i, (m, n) in enumerate(shapes):
        a, b = to64(out_ident[i][:, :n]), to64(out_bulk[i][:, :n])
        ref = O.newton_schulz(x64[i], 5)
        gate_bf16_ns(a, ref, x64[i], 5, what=f"identity form {m}x{n}")
        gate_bf16_ns(b, ref, x64[i], 5, what=f"bulk-load form {m}x{n}")
        assert rel(a, b) <= TOL_GPU_VS_GPU, f"identity vs bulk-load form {m}x{n}: {rel(a, b):.3e}"
    assert h.status() == (0, 0, 0)
    h.close()


def test_ns_zero_steps_scales(opt_bf16):
    shapes = [(10, 20), (20, 10)]
    xin, x64 = _ns_inputs(shapes, 9)
    sumsq = torch.tensor([np.sum(x ** 2) for x in x64], dtype=torch.float64, device=DEV)
    xout = [x_buffer(m, n) for (m, n) in shapes]
    opt_bf16.newton_schulz(xin, xout, shapes, sumsq, ns_steps=0)
    torch.cuda.synchronize()
    for i, (m, n) in enumerate(shapes):
        ref = O.newton_schulz(x64[i], 0)
        assert rel(to64(xout[i][:, :n]), ref) <= 4e-3


@pytest.mark.parametrize("steps", [1, 5])
def test_ns_fp32_matches_oracle(opt_fp32, steps):
    rng = np.random.default_rng(10)
    shapes = RAGGED
    xin, x64 = [], []
    for (m, n) in shapes:
        buf = x_buffer(m, n, torch.float32, fill=rng.standard_normal((m, n)))
        xin.append(buf)
        x64.append(to64(buf[:, :n]))
    sumsq = torch.tensor([np.sum(x ** 2) for x in x64], dtype=torch.float64, device=DEV)
    xout = [x_buffer(m, n, torch.float32) for (m, n) in shapes]
    opt_fp32.newton_schulz(xin, xout, shapes, sumsq, ns_steps=steps)
    torch.cuda.synchronize()
    for i, (m, n) in enumerate(shapes):
        ref = O.newton_schulz(x64[i], steps)
        got = to64(xout[i][:, :n])
        assert rel(got, ref) <= TOL_FP32_NS, f"matrix {i} {m}x{n}: {rel(got, ref):.3e}"


@pytest.mark.parametrize("kind", ["pair", "single"])
def test_ns_gram_upper_triangle_in_workspace(opts, kind):
    # The Gram tiles on and right of the 256-block diagonal hold the Gram of
    # the bf16 input at bf16 level; the diagonal blocks are exactly
    # symmetric. The single-CTA kernel stores only that upper 256-block
    # triangle (its consumers read the blocks below it transposed), the
    # CTA-pair kernel also writes the mirror image.
    from gpu_helpers import workspace_matrix
    opt_bf16 = opts[kind]
    shapes = [(600, 900), (900, 600), (513, 513), (1100, 300)]
    xin, x64 = _ns_inputs(shapes, 11, scale=0.03)
    xout = [x_buffer(m, n) for (m, n) in shapes]
    opt_bf16.newton_schulz(xin, xout, shapes, None, ns_steps=1)
    torch.cuda.synchronize()
    for i, (m, n) in enumerate(shapes):
        s = min(m, n)
        A = to64(workspace_matrix(opt_bf16, shapes, i, 2)[:, :s])
        blk = np.arange(s) // 256
        upper = blk[None, :] >= blk[:, None]          # stored: column block at or right of the row block
        full = np.where(upper, A, A.T)                 # the mirror image of the stored part
        X = x64[i] if m <= n else x64[i].T
        ref = X @ X.T
        assert rel(full, ref) <= 4e-3
        for b in range(0, s, 256):
            d = A[b:b + 256, b:b + 256]
            assert np.array_equal(d, d.T)
        if kind == "pair":
            assert np.array_equal(A, A.T)


SWEEP_POINTS = W.PARITY_SHAPES["sweep"]


@pytest.mark.parametrize("point", SWEEP_POINTS, ids=lambda p: f"{p[0]}x{p[1]}x{p[2]}")
def test_ns_only_sweep_inputs(opt_bf16, point):
    # NS-only workload: bf16 X with log-uniform singular values in [1e-4, 1],
    # no normalisation; five steps. The pages' own bf16 program lands far
    # above 2e-2 from exact on these inputs (small singular values grow by
    # the polynomial's slope a = 3.4445 per step, rounding noise with them):
    # its frozen distance is the gate.
    m, n, batch = point
    shapes = [(m, n)] * batch
    xin, x64 = [], []
    for b in range(batch):
        x = W.sweep_matrix(m, n, b)
        buf = x_buffer(m, n, fill=x)
        xin.append(buf)
        x64.append(to64(buf[:, :n]))
        assert np.array_equal(x64[-1], x)
    xout = [x_buffer(m, n) for _ in shapes]
    opt_bf16.newton_schulz(xin, xout, shapes, None, ns_steps=5)
    torch.cuda.synchronize()
    for b in range(batch):
        ref = O.ns_only(x64[b], 5)
        gate_bf16_ns(to64(xout[b][:, :n]), ref, x64[b], 5, normalised=False, what=f"config sweep {m}x{n} #{b}")
    _assert_status_clean(opt_bf16)


@pytest.mark.parametrize("kind", ["pair", "single"])
def test_ns_extreme_aspect_ratios(opts, kind):
    # Rows of a million elements (one K-block polynomial, a Gram over 16384
    # K-blocks), million-row combines, a ragged 70001-long row: five
    # normalised steps on the tiled phases against the oracle.
    opt_bf16 = opts[kind]
    shapes = W.PARITY_SHAPES["extreme"]
    xin, x64 = _ns_inputs(shapes, 60)
    sumsq = torch.tensor([np.sum(x ** 2) for x in x64], dtype=torch.float64, device=DEV)
    xout = [x_buffer(m, n) for (m, n) in shapes]
    opt_bf16.newton_schulz(xin, xout, shapes, sumsq, ns_steps=5)
    torch.cuda.synchronize()
    for i, (m, n) in enumerate(shapes):
        gate_bf16_ns(to64(xout[i][:, :n]), O.newton_schulz(x64[i], 5), x64[i], 5, what=f"{kind} {m}x{n}")
    _assert_status_clean(opt_bf16)


SMALL_SHAPES = W.PARITY_SHAPES["small"]


@pytest.mark.parametrize("steps", [1, 5])
def test_small_path_matches_oracle_and_tiled_path(opt_bf16, steps):
    # The on-chip small-matrix kernel (all iterations in one CTA) against the
    # oracle, and against the tiled phases on the same inputs.
    shapes = SMALL_SHAPES
    assert muon.plan_query(shapes)["small"] == list(range(len(shapes)))
    xin, x64 = _ns_inputs(shapes, 30 + steps)
    sumsq = torch.tensor([np.sum(x ** 2) for x in x64], dtype=torch.float64, device=DEV)
    out_small = [x_buffer(m, n) for (m, n) in shapes]
    out_tiled = [x_buffer(m, n) for (m, n) in shapes]
    opt_bf16.newton_schulz(xin, out_small, shapes, sumsq, ns_steps=steps)
    tiled = muon.Muon(device=0, small_path=False)
    tiled.newton_schulz(xin, out_tiled, shapes, sumsq, ns_steps=steps)
    torch.cuda.synchronize()
    assert opt_bf16.last_launch_count() == 1       # one launch for every small matrix
    for i, (m, n) in enumerate(shapes):
        got = to64(out_small[i][:, :n])
        ref = O.newton_schulz(x64[i], steps)
        gate_bf16_ns(got, ref, x64[i], steps, what=f"small path {m}x{n}")
        assert rel(got, to64(out_tiled[i][:, :n])) <= TOL_GPU_VS_GPU, f"small vs tiled {m}x{n}"
    _assert_status_clean(opt_bf16)
    assert tiled.status() == (0, 0, 0)
    tiled.close()


def test_small_path_identity_is_exact(opt_bf16):
    shapes = SMALL_SHAPES
    xin, x64 = _ns_inputs(shapes, 40)
    xout = [x_buffer(m, n) for (m, n) in shapes]
    opt_bf16.newton_schulz(xin, xout, shapes, None, ns_steps=3, coeffs=(1.0, 0.0, 0.0))
    torch.cuda.synchronize()
    for i, (m, n) in enumerate(shapes):
        assert np.array_equal(to64(xout[i][:, :n]), x64[i]), f"{m}x{n}"
