"""Pins for the float64 oracle: printed values, closed forms, invariants.

Every check here ties the oracle to something other than itself: numbers
printed on the pages (``tests/golden``), the SVD closed form of the
odd-polynomial lemma, the textbook convergent iterations, hand-unrolled
recurrences and library routines (numpy SVD, torch bf16 conversion).
"""

import json
import os

import numpy as np
import pytest

from oracle import muon_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "ns_scalar_facts.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _close_printed(x, entry_value, digits):
    # The page prints rounded or truncated decimals (0.5545 appears as
    # 0.554), so allow one unit of the last printed digit.
    return abs(x - entry_value) <= 10.0 ** (-digits) + 1e-12


def _haar(rng, n, k):
    """n x k matrix with orthonormal columns (QR of a Gaussian, sign fixed)."""
    q, r = np.linalg.qr(rng.standard_normal((n, k)))
    return q * np.sign(np.diag(r))


def _diag_ns(d, steps=5, coeffs=O.DEFAULT_COEFFS):
    """The oracle's matrix Newton-Schulz on diag(d): returns the diagonal."""
    out = O.newton_schulz(np.diag(d), steps, coeffs)
    return np.diag(out)


# ---------------------------------------------------------------------------
# Printed scalar facts ("About Muon: Why Not Adam", section "The iteration
# does not converge, and that is deliberate"), checked through the oracle's
# matrix iteration wherever possible.
# ---------------------------------------------------------------------------

def test_golden_coefficients_match_oracle_default():
    g = _golden()
    assert tuple(g["coeffs"]) == O.DEFAULT_COEFFS


def test_one_step_on_unit_matrix_gives_printed_p_of_1():
    g = _golden()["p_at_1"]
    # A 1x1 matrix normalises to 1/(1 + eps); one matrix step gives p(1).
    out = O.newton_schulz(np.array([[5.0]]), steps=1)[0, 0]
    assert _close_printed(out, g["value"], g["digits"])


def test_five_steps_on_small_singular_values_match_printed():
    g = _golden()
    # diag(d) with ||d|| = 1: the normalised singular values are d itself
    # (up to eps = 1e-7), so the output diagonal is p^5(d).
    small = np.array([1e-3, 1e-4])
    d = np.concatenate([[np.sqrt(1.0 - np.sum(small ** 2))], small])
    out = _diag_ns(d)
    e3, e4 = g["five_steps_from_1e-3"], g["five_steps_from_1e-4"]
    assert _close_printed(out[1], e3["value"], e3["digits"])
    assert _close_printed(out[2], e4["value"], e4["digits"])


def test_fixed_points_and_slopes_match_printed():
    g = _golden()
    a, b, c = O.DEFAULT_COEFFS
    # p(s) = s  <=>  c s^4 + b s^2 + (a - 1) = 0  (s != 0): a quadratic in s^2.
    disc = b * b - 4 * c * (a - 1)
    roots = sorted(np.sqrt([(-b - np.sqrt(disc)) / (2 * c), (-b + np.sqrt(disc)) / (2 * c)]))
    fp = g["fixed_points"]
    for r, v in zip(roots, fp["value"]):
        assert _close_printed(r, v, fp["digits"])
    # The oracle's matrix iteration leaves the fixed point inside (0, 1]
    # where it is: diag(r, sqrt(1 - r^2)) has unit norm, so one matrix step
    # maps the normalised singular value r to p(r) = r.
    r = roots[0]
    d = np.array([r, np.sqrt(1.0 - r * r)])
    assert abs(_diag_ns(d, steps=1)[0] - r) < 1e-6
    # Slope by central difference of the oracle's scalar map.
    sl = g["slope_at_fixed_points"]
    for r, v in zip(roots, sl["value"]):
        h = 1e-6
        slope = (O.ns_poly(r + h) - O.ns_poly(r - h)) / (2 * h)
        assert _close_printed(slope, v, sl["digits"])
    sz = g["slope_at_zero"]
    assert _close_printed((O.ns_poly(1e-7) - O.ns_poly(-1e-7)) / 2e-7, sz["value"], sz["digits"])


def test_maximum_on_unit_interval_matches_printed():
    g = _golden()
    s = np.linspace(0.0, 1.0, 2_000_001)
    v = O.ns_poly(s)
    mx, am = g["max_on_unit_interval"], g["argmax_on_unit_interval"]
    assert _close_printed(v.max(), mx["value"], mx["digits"])
    assert _close_printed(s[v.argmax()], am["value"], am["digits"])


def test_iterates_settle_in_printed_band():
    g = _golden()["cycle_band"]
    s = np.linspace(1e-3, 1.0, 2001)
    s = O.ns_poly_iterate(s, steps=200)
    lo, hi = np.inf, -np.inf
    for _ in range(200):
        s = O.ns_poly(s)
        lo, hi = min(lo, s.min()), max(hi, s.max())
    assert _close_printed(lo, g["value"][0], g["digits"])
    assert _close_printed(hi, g["value"][1], g["digits"])


# ---------------------------------------------------------------------------
# Odd-polynomial lemma: NS(G) = U diag(f(sigma / (||G|| + eps))) V^T
# ("About Muon: Why Not Adam", section "The lemma that makes it possible").
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("shape", [(3, 5), (8, 8), (16, 4), (33, 17), (1, 7), (7, 1), (40, 64)])
@pytest.mark.parametrize("steps", [0, 1, 5])
def test_ns_equals_svd_closed_form(shape, steps):
    rng = np.random.default_rng(hash(shape) % 2 ** 32 + steps)
    G = rng.standard_normal(shape)
    U, sig, Vt = np.linalg.svd(G, full_matrices=False)
    x = sig / (np.linalg.norm(G) + O.EPS)
    a, b, c = O.DEFAULT_COEFFS
    for _ in range(steps):          # scalar map, written independently here
        x = a * x + b * x ** 3 + c * x ** 5
    expect = (U * x) @ Vt
    got = O.newton_schulz(G, steps)
    assert np.max(np.abs(got - expect)) < 1e-12


@pytest.mark.parametrize("shape", [(12, 20), (20, 12), (16, 16)])
def test_singular_vectors_preserved(shape):
    rng = np.random.default_rng(7)
    G = rng.standard_normal(shape)
    U, sig, Vt = np.linalg.svd(G, full_matrices=False)
    D = U.T @ O.newton_schulz(G) @ Vt.T
    off = D - np.diag(np.diag(D))
    assert np.max(np.abs(off)) < 1e-12
    assert np.all(np.diag(D) > 0)


def test_rank_one_closed_form():
    rng = np.random.default_rng(3)
    x, y = rng.standard_normal(9), rng.standard_normal(13)
    G = 2.5 * np.outer(x, y)
    f1 = O.ns_poly_iterate(np.linalg.norm(G) / (np.linalg.norm(G) + O.EPS))
    expect = f1 * np.outer(x, y) / (np.linalg.norm(x) * np.linalg.norm(y))
    assert np.max(np.abs(O.newton_schulz(G) - expect)) < 1e-12


def test_scaled_orthogonal_closed_form():
    rng = np.random.default_rng(4)
    n = 24
    Q = _haar(rng, n, n)
    G = 3.0 * Q
    # ||G||_F = 3 sqrt(n): every normalised singular value is 3/(3 sqrt(n)+eps).
    f = O.ns_poly_iterate(3.0 / (3.0 * np.sqrt(n) + O.EPS))
    assert np.max(np.abs(O.newton_schulz(G) - f * Q)) < 1e-12


def test_diagonal_signs():
    d = np.array([0.5, -0.3, 0.2, -0.01])
    out = _diag_ns(d)
    assert np.all(np.sign(out) == np.sign(d))
    full = O.newton_schulz(np.diag(d))
    assert np.max(np.abs(full - np.diag(np.diag(full)))) == 0.0


# ---------------------------------------------------------------------------
# Textbook convergent members of the family reduce NS to the polar factor
# ("About Muon: Why Not Adam", section "The iteration does not converge, and
# that is deliberate"): cubic 1.5x - 0.5x^3 and quintic (15/8, -10/8, 3/8).
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("coeffs,steps", [((1.5, -0.5, 0.0), 60), ((15 / 8, -10 / 8, 3 / 8), 40)])
@pytest.mark.parametrize("shape", [(10, 16), (16, 10), (12, 12)])
def test_convergent_coefficients_give_polar_factor(coeffs, steps, shape):
    rng = np.random.default_rng(11)
    m, n = shape
    k = min(m, n)
    U, V = _haar(rng, m, k), _haar(rng, n, k)
    sig = np.linspace(1.0, 0.2, k)        # well conditioned
    G = (U * sig) @ V.T
    polar = U @ V.T
    got = O.newton_schulz(G, steps, coeffs)
    assert np.max(np.abs(got - polar)) < 1e-10
    # LMO optimality ("The spectral ball gives UV^T"): <G, UV^T> = sum sigma.
    assert abs(np.sum(G * got) - sig.sum()) < 1e-9
    # ||UV^T||_F^2 = min(m, n) ("Scaling answers Problem 1").
    assert abs(np.sum(got ** 2) - k) < 1e-9


# ---------------------------------------------------------------------------
# Invariances
# ---------------------------------------------------------------------------

def test_transpose_invariance():
    rng = np.random.default_rng(5)
    G = rng.standard_normal((9, 21))
    assert np.max(np.abs(O.newton_schulz(G.T) - O.newton_schulz(G).T)) < 1e-13


def test_scale_invariance_up_to_eps():
    # LMO(alpha G) = LMO(G) ("How Do We Turn It Into a Real Optimizer?").
    rng = np.random.default_rng(6)
    G = rng.standard_normal((9, 21))
    assert np.max(np.abs(O.newton_schulz(1e3 * G) - O.newton_schulz(G))) < 1e-6


def test_square_is_not_transposed_but_agrees():
    rng = np.random.default_rng(8)
    G = rng.standard_normal((15, 15))
    X = G / (np.linalg.norm(G) + O.EPS)
    alt = O.newton_schulz(X.T * (np.linalg.norm(G) + O.EPS)).T
    assert np.max(np.abs(O.newton_schulz(G) - alt)) < 1e-12


def test_zero_gradient_gives_zero_update():
    out = O.newton_schulz(np.zeros((4, 6)))
    assert np.all(out == 0.0)


def test_ns_only_matches_normalised_path():
    rng = np.random.default_rng(9)
    G = rng.standard_normal((6, 10))
    X = G / (np.linalg.norm(G) + O.EPS)
    assert np.max(np.abs(O.ns_only(X) - O.newton_schulz(G))) < 1e-14


# ---------------------------------------------------------------------------
# Momentum and Nesterov: hand-unrolled three-step recurrence from zero.
# ---------------------------------------------------------------------------

def test_momentum_nesterov_unrolled():
    rng = np.random.default_rng(10)
    beta = 0.95
    g1, g2, g3 = (rng.standard_normal((3, 4)) for _ in range(3))
    m = np.zeros((3, 4))
    m = O.momentum_update(m, g1, beta)
    u1 = O.nesterov_blend(g1, m, beta)
    assert np.allclose(m, (1 - beta) * g1, rtol=0, atol=1e-15)
    assert np.allclose(u1, (1 - beta ** 2) * g1, rtol=0, atol=1e-15)
    m = O.momentum_update(m, g2, beta)
    m2 = beta * (1 - beta) * g1 + (1 - beta) * g2
    assert np.allclose(m, m2, rtol=0, atol=1e-15)
    u2 = O.nesterov_blend(g2, m, beta)
    assert np.allclose(u2, (1 - beta) * g2 + beta * m2, rtol=0, atol=1e-15)
    m = O.momentum_update(m, g3, beta)
    m3 = beta ** 2 * (1 - beta) * g1 + beta * (1 - beta) * g2 + (1 - beta) * g3
    assert np.allclose(m, m3, rtol=0, atol=1e-15)
    u3 = O.nesterov_blend(g3, m, beta)
    assert np.allclose(u3, (1 - beta) * g3 + beta * m3, rtol=0, atol=1e-15)
    # Nesterov off: the update direction is the buffer itself.
    assert np.array_equal(O.nesterov_blend(g3, m, beta, nesterov=False), m)


def test_nesterov_off_beta_zero_is_plain_gradient():
    rng = np.random.default_rng(12)
    g = rng.standard_normal((5, 5))
    m = O.momentum_update(rng.standard_normal((5, 5)), g, 0.0)
    assert np.array_equal(O.nesterov_blend(g, m, 0.0, nesterov=False), g)


# ---------------------------------------------------------------------------
# Scale and apply
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("shape", [(64, 256), (256, 64), (128, 128)])
def test_moonlight_scale_gives_entry_rms_point_two(shape):
    # "Scaling answers Problem 1": 0.2 sqrt(max(m, n)) makes the entry RMS of
    # the scaled polar factor 0.2.
    rng = np.random.default_rng(13)
    m, n = shape
    k = min(m, n)
    polar = _haar(rng, m, k) @ _haar(rng, n, k).T
    lr = 1e-3
    p = rng.standard_normal(shape)
    scale = O.update_scale(m, n, O.SCALE_MOONLIGHT)
    dp = O.apply_update(p, polar, lr, 0.0, scale) - p
    rms = np.sqrt(np.mean(dp ** 2)) / lr
    assert abs(rms - 0.2) < 1e-12


def test_jordan_and_bernstein_scales():
    # "How Do We Turn It Into a Real Optimizer?": Jordan = Bernstein when
    # m >= n, Jordan = 1 when the layer shrinks (m < n).
    assert O.update_scale(64, 256, O.SCALE_JORDAN) == 1.0
    assert O.update_scale(256, 64, O.SCALE_JORDAN) == O.update_scale(256, 64, O.SCALE_BERNSTEIN) == 2.0
    # "The spectral ball gives UV^T": Bernstein's prefactor on a square layer is 1.
    assert O.update_scale(300, 300, O.SCALE_BERNSTEIN) == 1.0
    assert O.update_scale(300, 300, O.SCALE_MOONLIGHT) == pytest.approx(0.2 * np.sqrt(300), rel=1e-15)
    assert O.update_scale(5, 7, O.SCALE_NONE, 2.5) == 2.5


def test_weight_decay_alone():
    p = np.array([[1.0, -2.0], [3.0, 4.0]])
    out = O.apply_update(p, np.zeros_like(p), lr=0.1, wd=0.5, scale=3.0)
    assert np.allclose(out, p * 0.95, rtol=0, atol=1e-15)


def test_muon_step_skips_none_and_checks_2d():
    rng = np.random.default_rng(14)
    p = [rng.standard_normal((4, 6)), rng.standard_normal((6, 4))]
    m = [np.zeros((4, 6)), np.ones((6, 4))]
    g = [rng.standard_normal((4, 6)), None]
    P, M, Os, N = O.muon_step(p, g, m, lr=0.1)
    assert np.array_equal(P[1], p[1]) and np.array_equal(M[1], m[1])
    assert Os[1] is None and N[1] is None
    assert N[0] == pytest.approx(np.linalg.norm(O.nesterov_blend(g[0], M[0], 0.95)))
    with pytest.raises(ValueError):
        O.muon_step_matrix(np.zeros(3), np.zeros(3), np.zeros(3), lr=0.1)


def test_full_step_against_composed_closed_form():
    # p' = p(1 - lr wd) - lr*scale*U f^5(sigma_u/(||u||+eps)) V^T with u the
    # Nesterov blend of the hand-unrolled first step, u = (1 - beta^2) g.
    rng = np.random.default_rng(15)
    p, g = rng.standard_normal((6, 9)), rng.standard_normal((6, 9))
    beta, lr, wd = 0.9, 0.02, 0.1
    u = (1 - beta ** 2) * g
    U, sig, Vt = np.linalg.svd(u, full_matrices=False)
    x = sig / (np.linalg.norm(u) + O.EPS)
    a, b, c = O.DEFAULT_COEFFS
    for _ in range(5):
        x = a * x + b * x ** 3 + c * x ** 5
    expect = p * (1 - lr * wd) - lr * 0.2 * np.sqrt(9) * ((U * x) @ Vt)
    got, _, _, _ = O.muon_step_matrix(p, g, np.zeros_like(p), lr=lr, beta=beta, wd=wd)
    assert np.max(np.abs(got - expect)) < 1e-13


# ---------------------------------------------------------------------------
# bf16 rounding and the pages' bf16 program, against torch's bfloat16 tensors.
# ---------------------------------------------------------------------------

def test_bf16_round_matches_torch_on_float32_values():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(16)
    x = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-20, 20, 20000),
        # ties and near-ties around 1
        1.0 + np.arange(-64, 64) * 2.0 ** -9,
        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, np.inf, -np.inf]),
    ]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.bf16_round(x.astype(np.float64))
    assert np.array_equal(got, ref)


def test_bf16_ties_to_even():
    one = 1.0
    ulp = 2.0 ** -7
    assert O.bf16_round(np.array([one + ulp / 2]))[0] == one          # tie -> even
    assert O.bf16_round(np.array([one + 3 * ulp / 2]))[0] == one + 2 * ulp
    assert O.bf16_round(np.array([one + ulp / 2 + 1e-12]))[0] == one + ulp


def test_bf16_program_close_to_exact_but_rounded():
    # The pages' bf16 program on a well-conditioned input: a few bf16
    # roundings per operation, amplified by the polynomial's slopes, land a
    # few 1e-2 from exact; never zero and never order one.
    rng = np.random.default_rng(17)
    m, n = 48, 80
    G = (_haar(rng, m, m) * np.linspace(1, 0.05, m)) @ _haar(rng, n, m).T
    exact = O.newton_schulz(G)
    prog = O.newton_schulz(G, precision="bf16")
    assert np.array_equal(O.bf16_round(prog), prog)          # a bf16 tensor
    rel = np.linalg.norm(prog - exact) / np.linalg.norm(exact)
    assert 1e-3 < rel < 1e-1


@pytest.mark.parametrize("shape", [(6, 10), (10, 6), (9, 9)])
@pytest.mark.parametrize("steps", [0, 1, 5])
def test_bf16_program_is_exact_mode_plus_rounding(monkeypatch, shape, steps):
    # With rounding made the identity, the bf16 program is the exact
    # iteration to float64 accuracy: it adds roundings and nothing else.
    rng = np.random.default_rng(18)
    G = rng.standard_normal(shape)
    monkeypatch.setattr(O, "bf16_round", lambda v: np.asarray(v, dtype=np.float64))
    a = O.newton_schulz(G, steps, precision="bf16")
    b = O.ns_only(G * 0.1, steps, precision="bf16")
    monkeypatch.undo()
    assert np.max(np.abs(a - O.newton_schulz(G, steps))) < 1e-12
    assert np.max(np.abs(b - O.ns_only(G * 0.1, steps))) < 1e-12


def _torch_bf16_iteration(G, steps, normalise):
    """The iteration run by torch on a CPU bfloat16 tensor, one eager
    operation at a time (each returns bf16): the precision the oracle's
    bf16 mode restates."""
    torch = pytest.importorskip("torch")
    a, b, c = O.DEFAULT_COEFFS
    t = torch.from_numpy(G).to(torch.bfloat16)
    if normalise:
        t = t / (torch.linalg.vector_norm(t) + O.EPS)
    left = t.shape[0] <= t.shape[1]
    for _ in range(steps):
        gram = t @ t.mT if left else t.mT @ t
        poly = b * gram + c * (gram @ gram)
        t = a * t + (poly @ t if left else t @ poly)
    return t.to(torch.float64).numpy()


@pytest.mark.parametrize("shape", [(12, 20), (20, 12), (16, 16)])
def test_bf16_program_matches_torch_bf16_tensors(shape):
    # One step: every element equal to torch's, except where torch's float32
    # accumulation lands on the other side of a bf16 rounding boundary (rare,
    # one bf16 step at most). Five steps: the two stay far closer to each
    # other than to the exact result.
    rng = np.random.default_rng(40)
    G = O.bf16_round(rng.standard_normal(shape))
    one = O.newton_schulz(G, 1, precision="bf16")
    ref = _torch_bf16_iteration(G, 1, True)
    same = np.mean(one == ref)
    assert same >= 0.97, f"only {same:.3f} of the elements agree"
    assert np.all(np.abs(one - ref) <= 2.0 ** -7 * np.maximum(np.abs(ref), 2.0 ** -20))
    five = O.newton_schulz(G, 5, precision="bf16")
    ref5 = _torch_bf16_iteration(G, 5, True)
    exact = O.newton_schulz(G, 5)
    assert np.linalg.norm(five - ref5) < 0.5 * np.linalg.norm(five - exact)
    # Without the norm (NS-only inputs).
    X = O.bf16_round(G * 0.05)
    assert np.mean(O.ns_only(X, 1, precision="bf16") == _torch_bf16_iteration(X, 1, False)) >= 0.97


def test_bf16_program_norm_is_a_bf16_scalar():
    # The program divides by the bf16 norm of the bf16 copy plus eps (a bf16
    # scalar): the normalised matrix equals torch's bf16 division.
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(41)
    G = rng.standard_normal((33, 17)) * 3.0
    t = torch.from_numpy(G).to(torch.bfloat16)
    want = (t / (torch.linalg.vector_norm(t) + O.EPS)).to(torch.float64).numpy()
    got = O.newton_schulz(G, 0, precision="bf16")
    assert np.array_equal(got, want)


def test_precision_names_are_checked():
    with pytest.raises(ValueError):
        O.newton_schulz(np.eye(3), 1, precision="fp16")
    with pytest.raises(ValueError):
        O.muon_step_matrix(np.eye(3), np.eye(3), np.zeros((3, 3)), lr=0.1, gram=True, precision="bf16")


# ---------------------------------------------------------------------------
# Split Muon ("Why Muon Works", section 7.3; "The Optimizer Wars", Muon
# Split / Per-Head Muon): each row block is orthogonalised on its own.
# ---------------------------------------------------------------------------

def test_split_with_one_block_is_plain_step():
    rng = np.random.default_rng(21)
    p, g = rng.standard_normal((12, 20)), rng.standard_normal((12, 20))
    a = O.muon_step_matrix(p, g, np.zeros_like(p), lr=0.1)
    b = O.muon_step_matrix_split(p, g, np.zeros_like(p), [12], lr=0.1)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[2], b[2])


def test_split_blocks_follow_their_own_svd():
    # Every block of O equals U_h f^5(sigma_h / (||u_h|| + eps)) V_h^T of its
    # own block's SVD, and block norms are the blocks' own.
    rng = np.random.default_rng(22)
    g = rng.standard_normal((24, 16))
    blocks = [8, 8, 8]
    _, _, o, norms = O.muon_step_matrix_split(np.zeros_like(g), g, np.zeros_like(g), blocks, lr=0.1, beta=0.0,
                                              nesterov=False, wd=0.0)
    r0 = 0
    for h, nu in zip(blocks, norms):
        gb = g[r0:r0 + h]
        U, sig, Vt = np.linalg.svd(gb, full_matrices=False)
        x = sig / (np.linalg.norm(gb) + O.EPS)
        a, b, c = O.DEFAULT_COEFFS
        for _ in range(5):
            x = a * x + b * x ** 3 + c * x ** 5
        assert np.max(np.abs(o[r0:r0 + h] - (U * x) @ Vt)) < 1e-12
        assert abs(nu - np.linalg.norm(gb)) < 1e-12
        r0 += h
    # Not the same as orthogonalising the whole matrix.
    whole = O.newton_schulz(g)
    assert np.max(np.abs(whole - o)) > 1e-3


def test_split_rejects_bad_blocks():
    with pytest.raises(ValueError):
        O.muon_step_matrix_split(np.zeros((6, 4)), np.zeros((6, 4)), np.zeros((6, 4)), [4, 4], lr=0.1)


# ---------------------------------------------------------------------------
# Coefficient schedules: a sequence of odd polynomials still acts on the
# singular values only (lemma), and convergent members reach the polar factor.
# ---------------------------------------------------------------------------

def test_schedule_of_constant_rows_equals_triple():
    rng = np.random.default_rng(23)
    G = rng.standard_normal((10, 14))
    assert np.array_equal(O.newton_schulz(G, 4, [O.DEFAULT_COEFFS] * 4), O.newton_schulz(G, 4))


def test_schedule_follows_composed_scalar_polynomials():
    rng = np.random.default_rng(24)
    G = rng.standard_normal((9, 13))
    table = [(3.4445, -4.7750, 2.0315), (1.875, -1.25, 0.375), (1.5, -0.5, 0.0), (2.0, -1.5, 0.5)]
    U, sig, Vt = np.linalg.svd(G, full_matrices=False)
    x = sig / (np.linalg.norm(G) + O.EPS)
    for a, b, c in table:
        x = a * x + b * x ** 3 + c * x ** 5
    assert np.max(np.abs(O.newton_schulz(G, 4, table) - (U * x) @ Vt)) < 1e-12
    for precision in ("exact", "bf16"):
        with pytest.raises(ValueError):
            O.newton_schulz(G, 3, table, precision=precision)


def test_alternating_convergent_schedule_gives_polar_factor():
    rng = np.random.default_rng(25)
    U, V = _haar(rng, 12, 12), _haar(rng, 20, 12)
    G = (U * np.linspace(1.0, 0.3, 12)) @ V.T
    table = [(1.5, -0.5, 0.0), (15 / 8, -10 / 8, 3 / 8)] * 20
    assert np.max(np.abs(O.newton_schulz(G, 40, table) - U @ V.T)) < 1e-10


# ---------------------------------------------------------------------------
# QK-Clip ("The Optimizer Wars", MuonClip): the q.k logit of a clipped head
# scales by gamma_h = tau / S_max^h; other heads are untouched.
# ---------------------------------------------------------------------------

def test_qk_clip_scales_head_logits_by_gamma():
    rng = np.random.default_rng(26)
    heads, d, dm = 4, 8, 16
    wq, wk = rng.standard_normal((heads * d, dm)), rng.standard_normal((heads * d, dm))
    s_max = np.array([250.0, 50.0, 100.0, np.nan])
    tau = 100.0
    wq2, wk2 = O.qk_clip(wq, s_max, tau, d), O.qk_clip(wk, s_max, tau, d)
    x, y = rng.standard_normal(dm), rng.standard_normal(dm)
    for h in range(heads):
        sl = slice(h * d, (h + 1) * d)
        before = (wq[sl] @ x) @ (wk[sl] @ y)
        after = (wq2[sl] @ x) @ (wk2[sl] @ y)
        gamma = min(1.0, tau / s_max[h]) if np.isfinite(s_max[h]) else 1.0
        assert after == pytest.approx(gamma * before, rel=1e-12)
    assert np.array_equal(wq2[8:24], wq[8:24])


# ---------------------------------------------------------------------------
# Gram Newton-Schulz ("About Muon: Why Not Adam", section "Gram
# Newton-Schulz"): in exact arithmetic it returns the same matrix.
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("shape", [(3, 5), (8, 8), (16, 4), (33, 17), (20, 70), (1, 9)])
@pytest.mark.parametrize("steps", [0, 1, 2, 5])
@pytest.mark.parametrize("segment", [1, 2, None])
def test_gram_ns_equals_standard_ns(shape, steps, segment):
    rng = np.random.default_rng(hash(shape) % 2 ** 32 + 7 * steps)
    G = rng.standard_normal(shape)
    U, sig, Vt = np.linalg.svd(G, full_matrices=False)
    x = sig / (np.linalg.norm(G) + O.EPS)
    a, b, c = O.DEFAULT_COEFFS
    for _ in range(steps):
        x = a * x + b * x ** 3 + c * x ** 5
    got = O.gram_newton_schulz(G, steps, segment=segment)
    assert np.max(np.abs(got - (U * x) @ Vt)) < 1e-11
    assert np.max(np.abs(got - O.newton_schulz(G, steps))) < 1e-11


def test_gram_ns_with_schedule_and_steps():
    rng = np.random.default_rng(27)
    G = rng.standard_normal((12, 30))
    table = [(3.4445, -4.7750, 2.0315), (1.875, -1.25, 0.375), (1.5, -0.5, 0.0)]
    assert np.max(np.abs(O.gram_newton_schulz(G, 3, table) - O.newton_schulz(G, 3, table))) < 1e-11
    rng = np.random.default_rng(28)
    p, g = rng.standard_normal((10, 40)), rng.standard_normal((10, 40))
    r1 = O.muon_step_matrix(p, g, np.zeros_like(p), lr=0.1, gram=True)
    r2 = O.muon_step_matrix(p, g, np.zeros_like(p), lr=0.1)
    assert np.max(np.abs(r1[0] - r2[0])) < 1e-12
