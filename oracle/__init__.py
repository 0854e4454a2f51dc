"""Float64 CPU oracle for the Muon optimizer step.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import or run it. It shares no code with the CUDA path.

Modules
-------
muon_oracle
    The step itself, written from the pages in float64: momentum, Nesterov
    blend, Frobenius normalisation, the quintic Newton-Schulz iteration,
    the shape-dependent update scale, decoupled weight decay and the write.
plan_tables
    An independent restatement of the integer work lists (tile enumeration,
    workspace offsets) that the C++ plan builder produces, so the two can be
    compared bit for bit.

Parity status: every function in ``muon_oracle`` is pinned by a ``not gpu``
test (closed forms, SVD, printed scalar values, hand-unrolled recurrences).
The bf16-emulating mode of ``newton_schulz`` is a diagnostic, not a gate, and
is "parity unpinned" beyond its agreement with the exact mode at bf16 level.
"""

from .muon_oracle import (  # noqa: F401
    DEFAULT_COEFFS,
    EPS,
    SCALE_BERNSTEIN,
    SCALE_JORDAN,
    SCALE_MOONLIGHT,
    SCALE_NONE,
    apply_update,
    bf16_round,
    coeff_rows,
    gram_newton_schulz,
    momentum_update,
    muon_step,
    muon_step_matrix,
    muon_step_matrix_split,
    nesterov_blend,
    newton_schulz,
    ns_only,
    ns_poly,
    ns_poly_iterate,
    qk_clip,
    update_scale,
)
