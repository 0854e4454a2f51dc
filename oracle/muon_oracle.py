"""Float64 reference implementation of one Muon step (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module. It shares no code with the CUDA path.

Sources (web pages; cited by title and section):

* "About Muon: Why Not Adam" -- the authority on the arithmetic.
  - section "The whole thing, in about forty lines": the step order
    (momentum lerp, Nesterov lerp, bf16 cast, Frobenius normalisation with
    eps = 1e-7, short-side transpose, the quintic loop, cast back, scale,
    decoupled weight decay, write), default hyper-parameters and the
    Moonlight scale used by that program.
  - section "The lemma that makes it possible": an odd polynomial in X and
    X^T X acts on the singular values only.
  - section "The iteration does not converge, and that is deliberate":
    (a, b, c) = (3.4445, -4.7750, 2.0315) and the scalar facts used as pins.
  - section "How Do We Turn It Into a Real Optimizer?": the Jordan and
    Moonlight multipliers, (m, n) = (fan-out, fan-in) = p.shape.
  - section "The spectral ball gives UV^T": Bernstein's multiplier
    sqrt(fan-out / fan-in).
* "Por qué AdamW para entrenar modelos de lenguaje, y qué está cambiando",
  section "Momentum: recordar el paso anterior": Muon uses the Nesterov form.
* "The Optimizer Wars: How Muon Is Replacing Adam in Frontier AI Training",
  section "What is Muon? Momentum orthogonalized by Newton-Schulz": five
  quintic iterations in bf16 with the same coefficients.

Readings where the pages are silent or disagree (each also listed in the
design notes):

* Momentum is the exponential moving average ``m' = beta*m + (1-beta)*g``
  (the only program on the pages uses the lerp form), and the Nesterov blend
  uses the *updated* buffer: ``u = g + beta*(m' - g)``.
* Nesterov defaults to on; a flag turns it off (``u = m'``).
* The norm is taken of the float64 ``u``; eps = 1e-7 is added to the norm,
  not to its square.
* The short-side transpose is strict: only m > n is transposed.
* No bf16 rounding in the exact mode. ``emulate_bf16=True`` rounds X, A, B
  (round-to-nearest-even) at the points where the GPU rounds: the cast of
  u, and every Gram / polynomial / combine output. Diagnostic only.
* ``ns_steps = 0`` returns the normalised matrix.
"""

from __future__ import annotations

import numpy as np

# (a, b, c): "About Muon: Why Not Adam", section "The iteration does not
# converge, and that is deliberate"; the same triple in "The Optimizer Wars",
# section "What is Muon? Momentum orthogonalized by Newton-Schulz".
DEFAULT_COEFFS = (3.4445, -4.7750, 2.0315)

# Added to ||G||_F before dividing: "About Muon: Why Not Adam", section
# "The whole thing, in about forty lines".
EPS = 1e-7

SCALE_MOONLIGHT = 0   # 0.2 * sqrt(max(m, n))
SCALE_JORDAN = 1      # sqrt(max(1, m / n))
SCALE_BERNSTEIN = 2   # sqrt(m / n)  (fan-out / fan-in)
SCALE_NONE = 3        # 1


# ---------------------------------------------------------------------------
# bf16 rounding (used only by the emulating diagnostic mode)
# ---------------------------------------------------------------------------

def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (ties to even).

    bf16 keeps 8 significant bits (1 implicit + 7 stored) and float32's
    exponent range. Rounding is done directly on the float64 bit pattern
    (52 stored mantissa bits, of which the top 7 are kept), so there is no
    double rounding through float32. Values stay float64.
    """
    x = np.asarray(x, dtype=np.float64)
    bits = x.view(np.uint64).copy()
    drop = np.uint64(52 - 7)
    lsb = (bits >> drop) & np.uint64(1)
    bias = (np.uint64(1) << (drop - np.uint64(1))) - np.uint64(1) + lsb
    finite = np.isfinite(x)
    rounded = (bits + bias) & ~((np.uint64(1) << drop) - np.uint64(1))
    out = np.where(finite, rounded, bits).view(np.float64)
    return out


# ---------------------------------------------------------------------------
# Scalar polynomial ("About Muon: Why Not Adam", sections "The lemma that
# makes it possible" and "The iteration does not converge, and that is
# deliberate")
# ---------------------------------------------------------------------------

def ns_poly(s, coeffs=DEFAULT_COEFFS):
    """The odd quintic p(s) = a s + b s^3 + c s^5 applied to scalars."""
    a, b, c = coeffs
    s = np.asarray(s, dtype=np.float64)
    return a * s + b * s ** 3 + c * s ** 5


def ns_poly_iterate(s, steps=5, coeffs=DEFAULT_COEFFS):
    """p composed with itself ``steps`` times."""
    s = np.asarray(s, dtype=np.float64)
    for _ in range(steps):
        s = ns_poly(s, coeffs)
    return s


# ---------------------------------------------------------------------------
# Matrix Newton-Schulz
# ---------------------------------------------------------------------------

def _matmul(P, Q, accum_fp32):
    """P @ Q; with accum_fp32 the operands (bf16 values, exact in float32)
    are multiplied with float32 accumulation, as tensor cores accumulate."""
    if not accum_fp32:
        return P @ Q
    return (P.astype(np.float32) @ Q.astype(np.float32)).astype(np.float64)


def coeff_rows(coeffs, steps):
    """Per-step (a, b, c): one triple for every step, or a table of `steps`
    triples (a schedule of different odd polynomials, "About Muon: Why Not
    Adam", section "Gram Newton-Schulz": Chebyshev-type schemes compose
    different odd polynomials)."""
    arr = np.asarray(coeffs, dtype=np.float64)
    if arr.ndim == 1:
        if arr.shape != (3,):
            raise ValueError("coefficients must be (a, b, c) or a table of them")
        return [tuple(arr)] * steps
    if arr.shape != (steps, 3):
        raise ValueError(f"a coefficient table needs {steps} rows of (a, b, c)")
    return [tuple(r) for r in arr]


def _ns_iterations(X, steps, coeffs, emulate_bf16, accum_fp32=False, start=0):
    """Run the quintic iteration on a short-side-first matrix X (s x l).

    Each step forms the Gram A = X X^T, the polynomial B = bA + cA^2 and the
    combine X <- aX + BX. This equals aX + bX(X^T X) + cX(X^T X)^2 because
    (X X^T)^k X = X (X^T X)^k ("About Muon: Why Not Adam", section "The lemma
    that makes it possible"). ``coeffs`` holds one triple per step (see
    coeff_rows); steps ``start..steps-1`` are run.
    """
    rnd = bf16_round if emulate_bf16 else (lambda v: v)
    for k in range(start, steps):
        a, b, c = coeffs[k]
        A = rnd(_matmul(X, X.T, accum_fp32))
        B = rnd(b * A + c * _matmul(A, A, accum_fp32))
        X = rnd(a * X + _matmul(B, X, accum_fp32))
    return X


def newton_schulz(G, steps=5, coeffs=DEFAULT_COEFFS, eps=EPS,
                  emulate_bf16=False, accum_fp32=False):
    """Approximate orthogonal polar factor of G (float64).

    "About Muon: Why Not Adam", section "The whole thing, in about forty
    lines": normalise by the Frobenius norm plus eps so every singular value
    lies in (0, 1], work on the short side (transpose when rows > columns),
    iterate the quintic ``steps`` times, undo the transpose.

    With ``emulate_bf16`` the input is rounded to bf16 before normalising and
    the normalisation factor is applied exactly where the GPU applies it
    (inside the first Gram and first combine); otherwise no rounding happens.
    ``accum_fp32`` (with ``emulate_bf16``) accumulates the products in
    float32 instead of float64: a second, equally valid bf16 realization.
    """
    G = np.asarray(G, dtype=np.float64)
    if G.ndim != 2:
        raise ValueError("Newton-Schulz is defined for 2D matrices only")
    rows = coeff_rows(coeffs, steps)
    transposed = G.shape[0] > G.shape[1]
    if not emulate_bf16:
        X = G / (np.linalg.norm(G) + eps)
        if transposed:
            X = X.T
        X = _ns_iterations(X, steps, rows, False)
        return X.T if transposed else X

    # bf16-emulating diagnostic: Y = bf16(G); alpha = 1/(||G|| + eps) is
    # folded into the first Gram (alpha^2) and the first combine (alpha).
    alpha = 1.0 / (np.linalg.norm(G) + eps)
    Y = bf16_round(G)
    if transposed:
        Y = Y.T
    if steps == 0:
        X = alpha * Y
    else:
        a, b, c = rows[0]
        A = bf16_round(alpha * alpha * _matmul(Y, Y.T, accum_fp32))
        B = bf16_round(b * A + c * _matmul(A, A, accum_fp32))
        X = bf16_round(alpha * (a * Y + _matmul(B, Y, accum_fp32)))
        X = _ns_iterations(X, steps, rows, True, accum_fp32, start=1)
    return X.T if transposed else X


def gram_newton_schulz(G, steps=5, coeffs=DEFAULT_COEFFS, eps=EPS, emulate_bf16=False, accum_fp32=False,
                       segment=2):
    """Gram Newton-Schulz ("About Muon: Why Not Adam", section "Gram
    Newton-Schulz"): the same odd polynomial, iterated on the small Gram.

    With X the normalised short-side-first matrix, a segment of L steps
    forms A = X X^T once and then, for each step, B = bA + cA^2 (so the
    plain step is X <- (aI + B) X); the segment's product
    Q = (a_L I + B_L) ... (a_1 I + B_1) is applied to X at the end, and the
    Gram is carried between the steps of a segment as A <- P A P (the Gram
    of P X, P = aI + B commutes with A). In exact arithmetic every segment
    length gives ``newton_schulz``. Reading: segments of 2 steps (a fresh
    Gram every second step) keep bf16 rounding from accumulating in the
    carried Gram; ``segment=None`` runs all steps in one segment (exact mode
    only). The aI parts are never stored: with B0, B1 the two steps' B,
      R = a0 A + B0 A,   A1 = a0 R + R B0,
      Q - a0 a1 I = a1 B0 + a0 B1 + B1 B0,
      X' = a0 a1 X + (Q - a0 a1 I) X.
    With ``emulate_bf16`` each of A, B0, R, A1, B1, Q - a0 a1 I and X' is
    rounded to bf16 (the normalisation folded into the first segment's Gram
    as alpha^2 and its final product as alpha).
    """
    G = np.asarray(G, dtype=np.float64)
    if G.ndim != 2:
        raise ValueError("Newton-Schulz is defined for 2D matrices only")
    rows = coeff_rows(coeffs, steps)
    seg = steps if segment is None else int(segment)
    if emulate_bf16 and not 1 <= seg <= 2:
        raise ValueError("the bf16 mode restates segments of 1 or 2 steps")
    rnd = bf16_round if emulate_bf16 else (lambda v: v)
    acc = accum_fp32 and emulate_bf16
    transposed = G.shape[0] > G.shape[1]
    alpha = 1.0 / (np.linalg.norm(G) + eps)
    X = bf16_round(G) if emulate_bf16 else G
    if transposed:
        X = X.T
    if steps == 0:
        X = alpha * X
        return X.T if transposed else X
    k, sc = 0, alpha
    while k < steps:
        L = min(max(seg, 1), steps - k)
        A = rnd(sc * sc * _matmul(X, X.T, acc))
        if emulate_bf16 or L <= 2:
            a0, b0, c0 = rows[k]
            B0 = rnd(b0 * A + c0 * _matmul(A, A, acc))
            if L == 1:
                X = rnd(sc * (a0 * X + _matmul(B0, X, acc)))
            else:
                a1, b1, c1 = rows[k + 1]
                R = rnd(a0 * A + _matmul(B0, A, acc))
                A1 = rnd(a0 * R + _matmul(R, B0, acc))
                B1 = rnd(b1 * A1 + c1 * _matmul(A1, A1, acc))
                Qd = rnd(a1 * B0 + a0 * B1 + _matmul(B1, B0, acc))
                X = rnd(sc * (a0 * a1 * X + _matmul(Qd, X, acc)))
        else:
            eye = np.eye(A.shape[0])
            Q = None
            for j in range(L):
                a, b, c = rows[k + j]
                P = a * eye + b * A + c * (A @ A)
                Q = P if Q is None else P @ Q
                A = P @ A @ P
            X = sc * (Q @ X)
        k += L
        sc = 1.0
    return X.T if transposed else X


def ns_only(X, steps=5, coeffs=DEFAULT_COEFFS, emulate_bf16=False, accum_fp32=False):
    """The Newton-Schulz phases alone on an already-scaled X (no norm).

    Used for the NS-only sweep workload, whose inputs are generated with
    singular values already in [1e-4, 1]. Same orientation rule as
    ``newton_schulz``; with ``emulate_bf16`` the input and every Gram,
    polynomial and combine output are rounded to bf16.
    """
    X = np.asarray(X, dtype=np.float64)
    if emulate_bf16:
        X = bf16_round(X)
    transposed = X.shape[0] > X.shape[1]
    if transposed:
        X = X.T
    X = _ns_iterations(X, steps, coeff_rows(coeffs, steps), emulate_bf16, accum_fp32 and emulate_bf16)
    return X.T if transposed else X


# ---------------------------------------------------------------------------
# Momentum and Nesterov ("About Muon: Why Not Adam", section "The whole
# thing, in about forty lines"; Nesterov: "Por qué AdamW ...", section
# "Momentum: recordar el paso anterior")
# ---------------------------------------------------------------------------

def momentum_update(m, g, beta):
    """m' = m + (1 - beta)(g - m) = beta*m + (1 - beta)*g (in float64)."""
    m = np.asarray(m, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    return beta * m + (1.0 - beta) * g


def nesterov_blend(g, m_new, beta, nesterov=True):
    """u = g + beta*(m' - g) with Nesterov, else u = m'."""
    g = np.asarray(g, dtype=np.float64)
    m_new = np.asarray(m_new, dtype=np.float64)
    if not nesterov:
        return m_new.copy()
    return g + beta * (m_new - g)


# ---------------------------------------------------------------------------
# Update scale and apply
# ---------------------------------------------------------------------------

def update_scale(m, n, mode=SCALE_MOONLIGHT, extra_scale=1.0):
    """Shape multiplier for the orthogonalised update, (m, n) = p.shape.

    * Moonlight 0.2*sqrt(max(m, n)) -- "About Muon: Why Not Adam", sections
      "Scaling answers Problem 1" and "How Do We Turn It Into a Real
      Optimizer?"; it is the multiplier of the program in "The whole thing,
      in about forty lines".
    * Jordan sqrt(max(1, m/n)) -- same page, "How Do We Turn It Into a Real
      Optimizer?".
    * Bernstein sqrt(fan-out / fan-in) = sqrt(m/n) -- same page, "The
      spectral ball gives UV^T".
    * None: 1.
    ``extra_scale`` multiplies the result (the "extra scale factor" knob of
    the Megatron configuration in "Why Muon Works").
    """
    m = float(m)
    n = float(n)
    if mode == SCALE_MOONLIGHT:
        s = 0.2 * np.sqrt(max(m, n))
    elif mode == SCALE_JORDAN:
        s = np.sqrt(max(1.0, m / n))
    elif mode == SCALE_BERNSTEIN:
        s = np.sqrt(m / n)
    elif mode == SCALE_NONE:
        s = 1.0
    else:
        raise ValueError(f"unknown scale mode {mode}")
    return s * float(extra_scale)


def apply_update(p, O, lr, wd, scale):
    """p' = p*(1 - lr*wd) - lr*scale*O (decoupled weight decay, then the step).

    Both terms use the old p ("About Muon: Why Not Adam", section "The whole
    thing, in about forty lines").
    """
    p = np.asarray(p, dtype=np.float64)
    O = np.asarray(O, dtype=np.float64)
    return p * (1.0 - lr * wd) - lr * scale * O


# ---------------------------------------------------------------------------
# Whole step
# ---------------------------------------------------------------------------

def muon_step_matrix(p, g, m, *, lr, beta=0.95, nesterov=True, wd=0.1,
                     ns_steps=5, coeffs=DEFAULT_COEFFS,
                     scale_mode=SCALE_MOONLIGHT, extra_scale=1.0,
                     emulate_bf16=False, accum_fp32=False, gram=False):
    """One Muon step on one matrix. Returns (p', m', O, ||u||_F).

    ``gram`` selects the Gram form of Newton-Schulz (same result in exact
    arithmetic).

    Order: momentum, Nesterov blend, Newton-Schulz (normalise, orient,
    iterate, orient back), scale, decoupled weight decay, write.
    """
    p = np.asarray(p, dtype=np.float64)
    if p.ndim != 2:
        raise ValueError("Muon applies to 2D weight matrices only")
    m_new = momentum_update(m, g, beta)
    u = nesterov_blend(g, m_new, beta, nesterov)
    nu = float(np.linalg.norm(u))
    if gram:
        O = gram_newton_schulz(u, ns_steps, coeffs, EPS, emulate_bf16, accum_fp32)
    else:
        O = newton_schulz(u, ns_steps, coeffs, EPS, emulate_bf16, accum_fp32)
    scale = update_scale(p.shape[0], p.shape[1], scale_mode, extra_scale)
    p_new = apply_update(p, O, lr, wd, scale)
    return p_new, m_new, O, nu


def qk_clip(w, s_max, tau, head_rows):
    """QK-Clip on one projection weight (rows = heads x head_rows).

    "The Optimizer Wars", section on MuonClip: after the Muon update, a head
    whose largest attention logit S_max^h exceeded tau gets
    gamma_h = min(1, tau / S_max^h), applied as sqrt(gamma_h) to that head's
    rows of W_q and of W_k, so their product shrinks by gamma_h. Heads at or
    below tau (and non-finite S_max) are left unchanged.
    """
    w = np.asarray(w, dtype=np.float64).copy()
    s_max = np.asarray(s_max, dtype=np.float64)
    if w.shape[0] != head_rows * len(s_max):
        raise ValueError("rows must be heads x head_rows")
    for h, s in enumerate(s_max):
        if np.isfinite(s) and s > tau:
            w[h * head_rows:(h + 1) * head_rows] *= np.sqrt(tau / s)
    return w


def muon_step_matrix_split(p, g, m, row_blocks, **kw):
    """Split Muon on one matrix: each row block is a Muon matrix of its own.

    "Why Muon Works", section 7.3 (QKV / MLA split): orthogonalise Q, K, V,
    or each head's rows, separately and put the blocks back together; "The
    Optimizer Wars", "Muon Split" and "Per-Head Muon": the projection matrix
    is cut into per-head blocks before orthogonalisation. Reading: momentum,
    normalisation, Newton-Schulz, scale (from the block's own shape, which
    keeps Moonlight's entry RMS of 0.2) and the write all act per block.
    ``row_blocks`` lists the block heights (summing to the row count).
    Returns (p', m', O, norms) with O concatenated and one norm per block.
    """
    p = np.asarray(p, dtype=np.float64)
    if sum(row_blocks) != p.shape[0] or min(row_blocks) < 1:
        raise ValueError("row blocks must be positive and sum to the row count")
    outs = []
    r0 = 0
    for h in row_blocks:
        sl = slice(r0, r0 + h)
        outs.append(muon_step_matrix(p[sl], np.asarray(g)[sl], np.asarray(m)[sl], **kw))
        r0 += h
    return (np.concatenate([o[0] for o in outs]), np.concatenate([o[1] for o in outs]),
            np.concatenate([o[2] for o in outs]), [o[3] for o in outs])


def muon_step(params, grads, momenta, *, lr, beta=0.95, nesterov=True,
              wd=0.1, ns_steps=5, coeffs=DEFAULT_COEFFS,
              scale_mode=SCALE_MOONLIGHT, extra_scale=1.0,
              emulate_bf16=False):
    """One Muon step over a list of matrices, one at a time.

    A ``None`` gradient skips its matrix (parameter and momentum unchanged).
    Returns lists (params', momenta', O, norms); O and norm are None for
    skipped matrices.
    """
    out_p, out_m, out_o, out_n = [], [], [], []
    for p, g, m in zip(params, grads, momenta):
        if g is None:
            out_p.append(np.asarray(p, dtype=np.float64).copy())
            out_m.append(np.asarray(m, dtype=np.float64).copy())
            out_o.append(None)
            out_n.append(None)
            continue
        r = muon_step_matrix(p, g, m, lr=lr, beta=beta, nesterov=nesterov,
                             wd=wd, ns_steps=ns_steps, coeffs=coeffs,
                             scale_mode=scale_mode, extra_scale=extra_scale,
                             emulate_bf16=emulate_bf16)
        out_p.append(r[0])
        out_m.append(r[1])
        out_o.append(r[2])
        out_n.append(r[3])
    return out_p, out_m, out_o, out_n
