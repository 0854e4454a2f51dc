"""Write ``bf16_program_errors.json``: how far the pages' own bf16 program
lands from the exact result on every bf16 parity-test input.

"About Muon: Why Not Adam", section "The whole thing, in about forty
lines", runs Newton-Schulz on a bfloat16 tensor. The oracle restates that
precision (``precision="bf16"``: the cast, the bf16 norm, and a bf16 result
for every operation of a step). For each Newton-Schulz input of the GPU
parity tests this script records the relative Frobenius distance between
that program's output and the exact float64 output. The GPU tests require
the library to be no further from exact than max(2e-2, that distance): the
stated 2e-2 wherever the pages' program meets it, the program's own
distance where it does not.

Only ``oracle/`` and the seeded input recipes (``workloads``) are used.
Run from the repository root: ``python tests/golden/make_bf16_program_errors.py``
(about 10 minutes on 8 cores, most of it the 14336 x 4096 Llama matrix).
"""

import json
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import muon_oracle as O  # noqa: E402
import workloads as W  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "bf16_program_errors.json")
F32 = lambda v: float(np.float32(v))  # noqa: E731  (scalars as the kernels receive them)
BETA = F32(0.95)


def rel(a, b):
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


entries = {}


def record(label, x, steps=5, coeffs=O.DEFAULT_COEFFS, normalised=True):
    key = W.case_key(x, steps, coeffs, normalised)
    if key in entries:
        return
    t = time.time()
    if normalised:
        exact = O.newton_schulz(x, steps, coeffs)
        prog = O.newton_schulz(x, steps, coeffs, precision="bf16")
    else:
        exact = O.ns_only(x, steps, coeffs)
        prog = O.ns_only(x, steps, coeffs, precision="bf16")
    entries[key] = {"label": label, "err": rel(prog, exact)}
    if time.time() - t > 5:
        print(f"  {label}: {entries[key]['err']:.4e} ({time.time() - t:.0f} s)", flush=True)


def step_input(g, m0, beta=BETA, nesterov=True):
    """The Newton-Schulz input of a step: momentum, then the blend."""
    return O.nesterov_blend(g, O.momentum_update(m0, g, beta), beta, nesterov)


def shape_set(name, config, shapes, grad_bf16=False, steps=(5,), coeffs=O.DEFAULT_COEFFS, indices=None,
              seed_base=0):
    vals = W.set_values(config, shapes, grad_bf16, seed_base=seed_base, indices=indices)
    for i, (p, g, m0) in vals.items():
        u = step_input(g, m0)
        for k in steps:
            record(f"{name} #{i} {shapes[i][0]}x{shapes[i][1]} steps {k}", u, k, coeffs)


def main():
    P = W.PARITY_SHAPES
    # Stage tests: one step with isolating coefficients (no norm), normalised
    # 1, 2 and 5 steps, the NS-only sweep inputs, the small on-chip path.
    xs = W.gaussian_set(P["ragged"], 6, scale=0.05)
    for coeffs in [(0.0, 1.0, 0.0), (0.0, 0.0, 1.0), (0.5, -0.25, 0.125)]:
        for (m, n), x in zip(P["ragged"], xs):
            record(f"stage one step {coeffs} {m}x{n}", x, 1, coeffs, normalised=False)
    for steps in (1, 2, 5):
        for (m, n), x in zip(P["ragged"], W.gaussian_set(P["ragged"], 7 + steps)):
            record(f"stage {m}x{n} steps {steps}", x, steps)
    for (m, n, batch) in P["sweep"]:
        for b in range(batch):
            record(f"sweep {m}x{n} #{b}", W.sweep_matrix(m, n, b), 5, normalised=False)
    for steps in (1, 5):
        for (m, n), x in zip(P["small"], W.gaussian_set(P["small"], 30 + steps)):
            record(f"small path {m}x{n} steps {steps}", x, steps)
    # Extreme aspect ratios, normalised, five steps.
    for (m, n), x in zip(P["extreme"], W.gaussian_set(P["extreme"], 60)):
        record(f"extreme {m}x{n}", x, 5)
    # Allocation-free stage: two calls with fresh inputs.
    for call in range(2):
        for (m, n), x in zip(P["noalloc"], W.gaussian_set(P["noalloc"], call)):
            record(f"no-alloc call {call} {m}x{n}", x, 5)
            record(f"no-alloc call {call} {m}x{n} steps 1", x, 1)
    # Whole steps on shape sets (zero momentum, beta 0.95, Nesterov).
    shape_set("single", W.CONFIG_SINGLE, W.single_shapes())
    shape_set("gpt2", W.CONFIG_GPT2, W.gpt2_shapes())
    shape_set("wait", W.CONFIG_GPT2, P["wait"])
    shape_set("mixed", W.CONFIG_GPT2, P["mixed"])
    shape_set("gram", W.CONFIG_GPT2, P["gram"], steps=(5, 4, 1))
    shape_set("deterministic", W.CONFIG_GPT2, P["deterministic"])
    shape_set("layerwise", W.CONFIG_GPT2, P["layerwise"])
    table = [tuple(F32(v) for v in r) for r in W.SCHEDULE_TABLE]
    shape_set("schedule", W.CONFIG_GPT2, P["schedule"], steps=(4,), coeffs=table)
    vals = W.set_values(W.CONFIG_GPT2, P["split"], False)
    for i, (p, g, m0) in vals.items():
        rows = P["split"][i][0] if W.SPLIT_ROWS[i] is None else W.SPLIT_ROWS[i]
        u = step_input(g, m0)
        for r0 in range(0, u.shape[0], rows):
            record(f"split #{i} rows {r0}..{r0 + rows}", u[r0:r0 + rows], 5)
    # Zero gradient, warm momentum, beta 0.9, Nesterov off: u = 0.9 m0.
    rng = np.random.default_rng(21)
    zshapes = [(64, 96), (96, 64), (32, 32), (48, 80)]
    [rng.standard_normal(s) for s in zshapes]
    moms = [W.as_float32_values(rng.standard_normal(s) * 0.1) for s in zshapes]
    record("zero gradient 96x64", step_input(np.zeros(zshapes[1]), moms[1], F32(0.9), False), 5)
    # Full-size sets, sampled matrices.
    shape_set("moe", W.CONFIG_MOE, W.moe_shapes(), True, indices=W.MOE_SAMPLE)
    shape_set("llama", W.CONFIG_LLAMA, W.llama3_8b_shapes(), True, indices=W.LLAMA_SAMPLE)
    with open(OUT, "w") as f:
        json.dump({"source": "About Muon: Why Not Adam, section 'The whole thing, in about forty lines' "
                             "(its bf16 program, restated by oracle precision='bf16')",
                   "measure": "relative Frobenius distance of the bf16 program's output from the exact output",
                   "cases": dict(sorted(entries.items()))}, f, indent=1)
    print(f"wrote {len(entries)} cases to {OUT}")


if __name__ == "__main__":
    main()
