"""Planted mistakes in the oracle are caught by facts that do not come from it.

Each case edits one line of a copy of ``oracle/muon_oracle.py`` in memory
(the file itself is never touched), loads the copy as a separate module and
runs a set of checks built only from the pages' closed forms and from
library routines: the SVD form of the lemma ("About Muon: Why Not Adam",
"The lemma that makes it possible"), the hand-unrolled momentum and Nesterov
recurrences, the printed multipliers, decoupled weight decay, torch's bf16
cast and bf16 tensor arithmetic, transpose invariance and the QK-Clip closed
form. The unmodified
oracle passes every check; every planted mistake fails at least one.
"""

import os
import types

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = open(os.path.join(ROOT, "oracle", "muon_oracle.py")).read()

A_, B_, C_ = 3.4445, -4.7750, 2.0315


def _load(src):
    mod = types.ModuleType("oracle_copy")
    exec(compile(src, "oracle_copy", "exec"), mod.__dict__)
    return mod


def _f5(s, steps=5):
    for _ in range(steps):
        s = A_ * s + B_ * s ** 3 + C_ * s ** 5
    return s


def _rng_matrix(m, n, seed):
    return np.random.default_rng(seed).standard_normal((m, n))


# --- checks that do not use the oracle's own arithmetic ----------------------

def check_svd_closed_form(O):
    for (m, n), seed in (((3, 5), 1), ((8, 8), 2), ((6, 3), 3), ((16, 4), 4)):
        G = _rng_matrix(m, n, seed)
        U, s, Vt = np.linalg.svd(G, full_matrices=False)
        want = U @ np.diag(_f5(s / (np.linalg.norm(G) + 1e-7))) @ Vt
        got = O.newton_schulz(G, 5)
        if not np.allclose(got, want, rtol=0, atol=1e-10):
            return False
    return True


def check_momentum_recurrence(O):
    beta = 0.9
    g1, g2 = np.array([[1.0, -2.0]]), np.array([[0.5, 4.0]])
    m1 = O.momentum_update(np.zeros((1, 2)), g1, beta)
    u1 = O.nesterov_blend(g1, m1, beta)
    m2 = O.momentum_update(m1, g2, beta)
    u2 = O.nesterov_blend(g2, m2, beta)
    ok = np.allclose(m1, (1 - beta) * g1) and np.allclose(u1, (1 - beta ** 2) * g1)
    ok &= np.allclose(m2, beta * (1 - beta) * g1 + (1 - beta) * g2)
    ok &= np.allclose(u2, (1 - beta) * g2 + beta * m2)
    ok &= np.allclose(O.nesterov_blend(g2, m2, beta, nesterov=False), m2)
    return bool(ok)


def check_scales(O):
    return (np.isclose(O.update_scale(256, 512, O.SCALE_MOONLIGHT), 0.2 * np.sqrt(512))
            and np.isclose(O.update_scale(512, 256, O.SCALE_MOONLIGHT), 0.2 * np.sqrt(512))
            and np.isclose(O.update_scale(512, 128, O.SCALE_JORDAN), 2.0)
            and np.isclose(O.update_scale(128, 512, O.SCALE_JORDAN), 1.0)
            and np.isclose(O.update_scale(512, 128, O.SCALE_BERNSTEIN), 2.0)
            and np.isclose(O.update_scale(128, 512, O.SCALE_BERNSTEIN), 0.5)
            and np.isclose(O.update_scale(7, 9, O.SCALE_NONE, 3.0), 3.0))


def check_apply(O):
    p = np.array([[1.0, -2.0]])
    o = np.array([[1.0, 1.0]])
    return bool(np.allclose(O.apply_update(p, o, 0.1, 0.5, 2.0), p * (1 - 0.05) - 0.2 * o))


def check_bf16_round(O):
    x = np.random.default_rng(5).standard_normal(4096) * 10.0 ** np.random.default_rng(6).integers(-6, 6, 4096)
    # exact ties: halfway between neighbours with an even and an odd last bit
    ties = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(2 + 2.0 ** -7), 0.5 * (1 + 5 * 2.0 ** -8)])
    x = np.concatenate([x, ties])
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    return bool(np.array_equal(O.bf16_round(x), want))


def _torch_bf16_step(G):
    """One normalised step run by torch on CPU bfloat16 tensors (each eager
    operation returns bf16)."""
    a, b, c = A_, B_, C_
    t = torch.from_numpy(G).to(torch.bfloat16)
    t = t / (torch.linalg.vector_norm(t) + 1e-7)
    left = t.shape[0] <= t.shape[1]
    gram = t @ t.mT if left else t.mT @ t
    poly = b * gram + c * (gram @ gram)
    t = a * t + (poly @ t if left else t @ poly)
    return t.to(torch.float64).numpy()


def check_bf16_program(O):
    # The oracle's bf16 mode agrees with torch's bf16 tensors element by
    # element (up to rare float32-accumulation boundary cases).
    for shape, seed in (((12, 20), 13), ((20, 12), 14)):
        G = _rng_matrix(*shape, seed)
        if np.mean(O.newton_schulz(G, 1, precision="bf16") == _torch_bf16_step(G)) < 0.97:
            return False
    for seed in range(15, 21):   # the normalisation alone: bf16 norm, bf16 division
        G = _rng_matrix(9, 11, seed) * 2.0 ** seed
        t = torch.from_numpy(G).to(torch.bfloat16)
        want = (t / (torch.linalg.vector_norm(t) + 1e-7)).to(torch.float64).numpy()
        if not np.array_equal(O.newton_schulz(G, 0, precision="bf16"), want):
            return False
    return True


def check_transpose(O):
    G = _rng_matrix(5, 3, 7)
    return bool(np.allclose(O.newton_schulz(G.T), O.newton_schulz(G).T, atol=1e-12))


def check_gram_form(O):
    for (m, n), seed in (((4, 9), 8), ((9, 4), 9)):
        G = _rng_matrix(m, n, seed)
        U, s, Vt = np.linalg.svd(G, full_matrices=False)
        want = U @ np.diag(_f5(s / (np.linalg.norm(G) + 1e-7))) @ Vt
        for seg in (1, 2, None):
            if not np.allclose(O.gram_newton_schulz(G, 5, segment=seg), want, rtol=0, atol=1e-9):
                return False
    return True


def check_qk_clip(O):
    w = np.ones((4, 3))
    got = O.qk_clip(w, [50.0, 400.0], 100.0, 2)
    want = np.vstack([np.ones((2, 3)), np.full((2, 3), np.sqrt(100.0 / 400.0))])
    return bool(np.allclose(got, want))


def check_whole_step(O):
    # Warm momentum, beta 0.9, wd 0, no scale: m' = beta m + (1 - beta) g,
    # u = g + beta (m' - g), p' = p - lr * NS(u) with NS from the SVD.
    p = _rng_matrix(4, 6, 10)
    g = _rng_matrix(4, 6, 11)
    m = _rng_matrix(4, 6, 12)
    beta = 0.9
    p2, m2, o, nu = O.muon_step_matrix(p, g, m, lr=0.5, beta=beta, wd=0.0, scale_mode=O.SCALE_NONE)
    m_want = beta * m + (1 - beta) * g
    u = g + beta * (m_want - g)
    U, s, Vt = np.linalg.svd(u, full_matrices=False)
    want_o = U @ np.diag(_f5(s / (np.linalg.norm(u) + 1e-7))) @ Vt
    return bool(np.allclose(o, want_o, atol=1e-10) and np.allclose(p2, p - 0.5 * want_o, atol=1e-10)
                and np.isclose(nu, np.linalg.norm(u)) and np.allclose(m2, m_want))


CHECKS = [check_svd_closed_form, check_momentum_recurrence, check_scales, check_apply, check_bf16_round,
          check_bf16_program, check_transpose, check_gram_form, check_qk_clip, check_whole_step]

MUTANTS = {
    "gram_of_columns_for_square": ("    return X @ X.T if X.shape[0] <= X.shape[1] else X.T @ X",
                                   "    return X @ X.T if X.shape[0] < X.shape[1] else X.T @ X"),
    "combine_side_for_square": ("    return P @ X if X.shape[0] <= X.shape[1] else X @ P",
                                "    return P @ X if X.shape[0] < X.shape[1] else X @ P"),
    "tall_uses_left_gram": ("    return X @ X.T if X.shape[0] <= X.shape[1] else X.T @ X",
                            "    return X @ X.T"),
    "sign_of_b": ("    B = b * A + c * (A @ A)\n    return a * X", "    B = -b * A + c * (A @ A)\n    return a * X"),
    "dropped_c": ("    B = b * A + c * (A @ A)\n    return a * X", "    B = b * A\n    return a * X"),
    "combine_drops_a": ("    return a * X + _on_short_side(B, X)", "    return X + _on_short_side(B, X)"),
    "eps_in_square": ("    return G / (np.linalg.norm(G) + eps)", "    return G / np.sqrt(np.linalg.norm(G) ** 2 + eps)"),
    "norm_squared": ("    return G / (np.linalg.norm(G) + eps)", "    return G / (np.linalg.norm(G) ** 2 + eps)"),
    "bf16_divisor_unrounded": ("    return bf16_round(Y / bf16_round(nrm + eps))",
                               "    return bf16_round(Y / (np.linalg.norm(Y) + eps))"),
    "bf16_gram_unrounded": ("    A = r(_short_gram(X))", "    A = _short_gram(X)"),
    "bf16_poly_fused": ("    B = r(r(b * A) + r(c * AA))", "    B = r(b * A + c * AA)"),
    "bf16_combine_fused": ("    return r(r(a * X) + BX)", "    return r(a * X + BX)"),
    "nesterov_wrong_base": ("    return g + beta * (m_new - g)", "    return m_new + beta * (m_new - g)"),
    "classic_momentum": ("    return beta * m + (1.0 - beta) * g", "    return beta * m + g"),
    "decay_scaled": ("    return p * (1.0 - lr * wd) - lr * scale * O", "    return p * (1.0 - lr * wd * scale) - lr * scale * O"),
    "decay_missing_lr": ("    return p * (1.0 - lr * wd) - lr * scale * O", "    return p * (1.0 - wd) - lr * scale * O"),
    "moonlight_min": ("        s = 0.2 * np.sqrt(max(m, n))", "        s = 0.2 * np.sqrt(min(m, n))"),
    "jordan_inverted": ("        s = np.sqrt(max(1.0, m / n))", "        s = np.sqrt(max(1.0, n / m))"),
    "bernstein_inverted": ("        s = np.sqrt(m / n)\n", "        s = np.sqrt(n / m)\n"),
    "bf16_truncates": ("    bias = (np.uint64(1) << (drop - np.uint64(1))) - np.uint64(1) + lsb",
                       "    bias = np.uint64(0) * lsb"),
    "bf16_ties_away": ("    bias = (np.uint64(1) << (drop - np.uint64(1))) - np.uint64(1) + lsb",
                       "    bias = (np.uint64(1) << (drop - np.uint64(1))) + np.uint64(0) * lsb"),
    "gram_form_no_carry": ("            A = P @ A @ P\n", "            A = A\n"),
    "gram_form_half_carry": ("            A = P @ A @ P\n", "            A = P @ A\n"),
    "qk_clip_without_sqrt": ("            w[h * head_rows:(h + 1) * head_rows] *= np.sqrt(tau / s)",
                             "            w[h * head_rows:(h + 1) * head_rows] *= tau / s"),
    "step_skips_nesterov": ("    u = nesterov_blend(g, m_new, beta, nesterov)\n    nu",
                            "    u = m_new\n    nu"),
}


def test_unmodified_oracle_passes_every_check():
    O = _load(SRC)
    for chk in CHECKS:
        assert chk(O), chk.__name__


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    old, new = MUTANTS[name]
    assert SRC.count(old) == 1, f"anchor of {name} not found once in the oracle"
    O = _load(SRC.replace(old, new))
    failed = []
    for chk in CHECKS:
        try:
            ok = chk(O)
        except Exception:   # a crash also counts as caught
            ok = False
        if not ok:
            failed.append(chk.__name__)
    assert failed, f"mutant {name} passed every check"
