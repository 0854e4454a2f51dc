"""Float64 reference implementation of one Muon step (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module. It shares no code with the CUDA path.

Sources (web pages; cited by title and section):

* "About Muon: Why Not Adam" -- the authority on the arithmetic.
  - section "The whole thing, in about forty lines": the step order
    (momentum lerp, Nesterov lerp, Frobenius normalisation with eps = 1e-7,
    the quintic iteration on the short side, scale, decoupled weight decay,
    write), default hyper-parameters, the Moonlight scale used by that
    program, and the precision of its iteration (a bf16 tensor, so every
    operation returns bf16).
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
* The short side is chosen by a strict test: only rows > columns works with
  X^T X (from the right); a square matrix uses X X^T (from the left). No
  transpose is formed: the two forms are the same matrix.
* ``precision="exact"`` (the default) rounds nothing. ``precision="bf16"``
  rounds to bf16 (round-to-nearest-even) wherever the pages' bf16 program
  returns a bf16 tensor: the cast of the input, its norm, norm + eps, the
  normalised matrix, and each of the eight operations of a step. It is the
  yardstick for how far bf16 arithmetic itself lands from the exact result.
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
# bf16 rounding (the precision of the pages' bf16 program)
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
#
# The lemma ("About Muon: Why Not Adam", section "The lemma that makes it
# possible"): for X = U S V^T, an odd polynomial written with the Gram of
# either side, a X + b (X X^T) X + c (X X^T)^2 X = a X + b X (X^T X) +
# c X (X^T X)^2, equals U p(S) V^T with p(s) = a s + b s^3 + c s^5. The
# work is cheapest with the s x s Gram of the short side, s = min(rows, cols):
# X X^T multiplied from the left when rows <= cols, X^T X from the right when
# rows > cols. That choice is the pages' "run on the short side" rule (a
# strict rows > cols test, so a square matrix takes the left form) written
# without transposing the matrix: the two forms are the same matrix.


def _short_gram(X):
    """The s x s Gram of the short side: X X^T (rows <= cols) or X^T X."""
    return X @ X.T if X.shape[0] <= X.shape[1] else X.T @ X


def _on_short_side(P, X):
    """P (s x s) applied on the short side: P X (rows <= cols) or X P."""
    return P @ X if X.shape[0] <= X.shape[1] else X @ P


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


def quintic_map(X, a, b, c):
    """p(X) = a X + b A X + c A^2 X in float64, A the short-side Gram.

    Evaluated in the pages' order: the Gram A, the polynomial part
    B = b A + c A^2, then the combine a X + B X (B acting on the short
    side).
    """
    A = _short_gram(X)
    B = b * A + c * (A @ A)
    return a * X + _on_short_side(B, X)


def quintic_map_bf16(X, a, b, c):
    """The same map at the precision of the pages' bf16 program.

    "About Muon: Why Not Adam", section "The whole thing, in about forty
    lines", runs the iteration on a bfloat16 tensor with plain tensor
    operations, so every operation returns a bf16 tensor: the Gram, the
    product A A, the scalings b A, c A^2 and a X, the sum that forms B, the
    product B X and the final sum. Each of those eight results is rounded to
    bf16 here. Reading: a bf16 matrix product is its exact value rounded once
    (accumulation in float32 on the devices that run such programs adds
    error far below one bf16 rounding), and a scalar times a bf16 tensor is
    the exact product rounded once.
    """
    r = bf16_round
    A = r(_short_gram(X))
    AA = r(A @ A)
    B = r(r(b * A) + r(c * AA))
    BX = r(_on_short_side(B, X))
    return r(r(a * X) + BX)


def frobenius_normalise(G, eps=EPS):
    """G / (||G||_F + eps): every singular value lands in [0, 1)."""
    G = np.asarray(G, dtype=np.float64)
    return G / (np.linalg.norm(G) + eps)


def frobenius_normalise_bf16(G, eps=EPS):
    """The normalisation of the pages' bf16 program: the matrix is cast to
    bf16 first, its norm is a bf16 scalar, adding eps rounds again, and the
    division returns a bf16 tensor."""
    Y = bf16_round(G)
    nrm = bf16_round(np.sqrt(np.sum(Y * Y)))
    return bf16_round(Y / bf16_round(nrm + eps))


PRECISIONS = ("exact", "bf16")


def _check_precision(precision):
    if precision not in PRECISIONS:
        raise ValueError(f"precision must be one of {PRECISIONS}")


def newton_schulz(G, steps=5, coeffs=DEFAULT_COEFFS, eps=EPS, precision="exact"):
    """Approximate orthogonal polar factor of G.

    Normalise by the Frobenius norm plus eps, then apply the quintic map
    ``steps`` times with the short-side Gram ("About Muon: Why Not Adam",
    sections "The whole thing, in about forty lines" and "The lemma that
    makes it possible"). ``precision="exact"`` works in float64 without any
    rounding; ``precision="bf16"`` rounds where the pages' bf16 program
    rounds (``frobenius_normalise_bf16``, ``quintic_map_bf16``). Zero steps
    return the normalised matrix.
    """
    G = np.asarray(G, dtype=np.float64)
    if G.ndim != 2:
        raise ValueError("Newton-Schulz is defined for 2D matrices only")
    _check_precision(precision)
    rows = coeff_rows(coeffs, steps)
    if precision == "exact":
        X, step = frobenius_normalise(G, eps), quintic_map
    else:
        X, step = frobenius_normalise_bf16(G, eps), quintic_map_bf16
    for a, b, c in rows:
        X = step(X, a, b, c)
    return X


def gram_newton_schulz(G, steps=5, coeffs=DEFAULT_COEFFS, eps=EPS, segment=2):
    """Gram Newton-Schulz ("About Muon: Why Not Adam", section "Gram
    Newton-Schulz"): the same odd polynomial, iterated on the small Gram.

    With X the normalised matrix and A its short-side Gram, one step is
    X <- P X with P = a I + b A + c A^2 (P on the short side), and the Gram
    of P X is P A P (P commutes with A). A segment of L steps forms A once,
    then for each step builds P from the carried Gram, accumulates the
    product Q = P_L ... P_1 and carries A <- P A P; the segment ends with
    X <- Q X. In exact arithmetic every segment length gives
    ``newton_schulz``. Reading: segments of 2 steps (a fresh Gram every
    second step), which is what keeps bf16 rounding from building up in the
    carried Gram; ``segment=None`` runs all steps in one segment.
    """
    G = np.asarray(G, dtype=np.float64)
    if G.ndim != 2:
        raise ValueError("Newton-Schulz is defined for 2D matrices only")
    rows = coeff_rows(coeffs, steps)
    seg = steps if segment is None else int(segment)
    if seg < 1 and steps > 0:
        raise ValueError("segments hold at least one step")
    X = frobenius_normalise(G, eps)
    k = 0
    while k < steps:
        A = _short_gram(X)
        eye = np.eye(A.shape[0])
        Q = eye
        for a, b, c in rows[k:k + seg]:
            P = a * eye + b * A + c * (A @ A)
            Q = P @ Q
            A = P @ A @ P
        X = _on_short_side(Q, X)
        k += seg
    return X


def ns_only(X, steps=5, coeffs=DEFAULT_COEFFS, precision="exact"):
    """The Newton-Schulz iterations alone on an already-scaled X (no norm).

    For the NS-only sweep, whose inputs are generated with singular values
    already in [1e-4, 1]. With ``precision="bf16"`` the input is cast to
    bf16 and each step rounds as the pages' bf16 program does.
    """
    X = np.asarray(X, dtype=np.float64)
    if X.ndim != 2:
        raise ValueError("Newton-Schulz is defined for 2D matrices only")
    _check_precision(precision)
    step = quintic_map if precision == "exact" else quintic_map_bf16
    if precision == "bf16":
        X = bf16_round(X)
    for a, b, c in coeff_rows(coeffs, steps):
        X = step(X, a, b, c)
    return X


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
                     precision="exact", gram=False):
    """One Muon step on one matrix. Returns (p', m', O, ||u||_F).

    ``gram`` selects the Gram form of Newton-Schulz (same result in exact
    arithmetic; exact precision only). ``precision`` is the Newton-Schulz
    precision ("exact" or the pages' "bf16" program); the momentum, blend,
    scale and write are float64 in both.

    Order: momentum, Nesterov blend, Newton-Schulz (normalise, iterate on
    the short side), scale, decoupled weight decay, write.
    """
    p = np.asarray(p, dtype=np.float64)
    if p.ndim != 2:
        raise ValueError("Muon applies to 2D weight matrices only")
    m_new = momentum_update(m, g, beta)
    u = nesterov_blend(g, m_new, beta, nesterov)
    nu = float(np.linalg.norm(u))
    if gram:
        if precision != "exact":
            raise ValueError("the Gram form is restated in exact arithmetic only")
        O = gram_newton_schulz(u, ns_steps, coeffs, EPS)
    else:
        O = newton_schulz(u, ns_steps, coeffs, EPS, precision)
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
              precision="exact"):
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
                             precision=precision)
        out_p.append(r[0])
        out_m.append(r[1])
        out_o.append(r[2])
        out_n.append(r[3])
    return out_p, out_m, out_o, out_n
