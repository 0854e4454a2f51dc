"""Seeded synthetic inputs for the Muon step (no arithmetic of the method).

Shared by the tests, ``bench.py`` and the CPU baseline. It produces matrices
with prescribed singular spectra and the shape sets of the workloads; it
computes nothing that the Muon step computes.

Shape sets (m, n) = (fan-out, fan-in), the PyTorch layout of a weight:
  * single : one 256 x 512 gradient
  * gpt2   : 12 layers x {QKV 2304x768, O 768x768, MLP up 3072x768,
             down 768x3072}                                  (48 matrices)
  * llama3 : 32 layers x {q 4096x4096, k 1024x4096, v 1024x4096,
             o 4096x4096, gate 14336x4096, up 14336x4096,
             down 4096x14336}                                 (224 matrices)
  * moe    : 128 experts x {gate 2048x7168, up 2048x7168, down 7168x2048}
                                                              (384 matrices)
  * sweep  : NS-only points, each side a power of two in [128, 16384],
             aspects 1:1, 1:4, 4:1, 1:8, batches 1..256.

Spectra:
  * power law s_i = i^-1.5 (+ 1e-3 N(0,1) noise); for the GPT-2 set the
    power law is cut at rank 64 ("low-rank power-law plus noise"); for the
    large sets it is cut at rank 512 (s_512 < 1e-4, far below the noise
    floor of a 1e-3 N(0,1) matrix of these sizes, whose singular values are
    ~1e-3 (sqrt(m) + sqrt(n)) > 0.1).
  * MoE: s_i = 10^(-4 (i-1)/(s-1)), i = 1..s (condition number 1e4), no noise.
  * sweep: log10 s_i uniform on [-4, 0].
Seeds: 1_000_000 * config + 1000 * layer + matrix_index (+ expert).
U, V: Haar orthonormal factors (QR of a Gaussian with the sign fix).
"""

from __future__ import annotations

import math

import numpy as np

CONFIG_SINGLE, CONFIG_GPT2, CONFIG_LLAMA, CONFIG_MOE, CONFIG_SWEEP = 1, 2, 3, 4, 5


# ---------------------------------------------------------------------------
# Shape sets
# ---------------------------------------------------------------------------

def single_shapes():
    return [(256, 512)]


def gpt2_shapes():
    out = []
    for _ in range(12):
        out += [(2304, 768), (768, 768), (3072, 768), (768, 3072)]
    return out


def llama3_8b_shapes():
    out = []
    for _ in range(32):
        out += [(4096, 4096), (1024, 4096), (1024, 4096), (4096, 4096), (14336, 4096), (14336, 4096),
                (4096, 14336)]
    return out


def llama3_layer_shapes():
    """One layer of the Llama-3-8B set (7 matrices): the small profiling case."""
    return llama3_8b_shapes()[:7]


def moe_shapes(experts: int = 128):
    out = []
    for _ in range(experts):
        out += [(2048, 7168), (2048, 7168), (7168, 2048)]
    return out


def sweep_points(max_bytes: float = 120e9):
    """NS-only sweep points (m, n, batch), skipping points above max_bytes."""
    pts = []
    sides = [2 ** k for k in range(7, 15)]
    for aspect in ("1:1", "1:4", "4:1", "1:8"):
        for s in sides:
            if aspect == "1:1":
                m, n = s, s
            elif aspect == "1:4":
                m, n = s, 4 * s
            elif aspect == "4:1":
                m, n = 4 * s, s
            else:
                m, n = s, 8 * s
            if max(m, n) > 16384:
                continue
            for batch in (1, 4, 16, 64, 256):
                sm = min(m, n)
                if batch * (3 * m * n + 2 * sm * sm) * 2 > max_bytes:
                    continue
                pts.append((m, n, batch))
    return pts


def seed_for(config: int, layer: int, index: int, expert: int = 0) -> int:
    return 1_000_000 * config + 1000 * layer + index + expert


# ---------------------------------------------------------------------------
# Spectra
# ---------------------------------------------------------------------------

def power_law(k: int, exponent: float = 1.5):
    return np.arange(1, k + 1, dtype=np.float64) ** (-exponent)


def log_spaced(k: int, decades: float = 4.0):
    if k == 1:
        return np.ones(1)
    return 10.0 ** (-decades * np.arange(k, dtype=np.float64) / (k - 1))


def log_uniform(rng, k: int, lo: float = -4.0, hi: float = 0.0):
    return np.sort(10.0 ** rng.uniform(lo, hi, size=k))[::-1]


# ---------------------------------------------------------------------------
# CPU generators (float64, numpy)
# ---------------------------------------------------------------------------

def haar(rng, n: int, k: int):
    """n x k with orthonormal columns, Haar distributed (QR + sign fix)."""
    q, r = np.linalg.qr(rng.standard_normal((n, k)))
    return q * np.sign(np.diag(r))


def spectral_matrix(m: int, n: int, sigma, seed: int, noise: float = 0.0):
    """U diag(sigma) V^T + noise * N(0, 1), float64, with rank len(sigma)."""
    rng = np.random.default_rng(seed)
    k = len(sigma)
    U = haar(rng, m, k)
    V = haar(rng, n, k)
    G = (U * np.asarray(sigma)) @ V.T
    if noise:
        G = G + noise * rng.standard_normal((m, n))
    return G


def gradient_cpu(config: int, m: int, n: int, seed: int):
    """float64 gradient of the config's recipe."""
    s = min(m, n)
    if config == CONFIG_SINGLE:
        return spectral_matrix(m, n, power_law(s), seed, noise=1e-3)
    if config == CONFIG_GPT2:
        return spectral_matrix(m, n, power_law(min(64, s)), seed, noise=1e-3)
    if config == CONFIG_LLAMA:
        return spectral_matrix(m, n, power_law(min(512, s)), seed, noise=1e-3)
    if config == CONFIG_MOE:
        return spectral_matrix(m, n, log_spaced(s), seed, noise=0.0)
    if config == CONFIG_SWEEP:
        rng = np.random.default_rng(seed + 7)
        return spectral_matrix(m, n, log_uniform(rng, s), seed, noise=0.0)
    raise ValueError(config)


def param_cpu(m: int, n: int, seed: int, std: float = 0.02):
    return std * np.random.default_rng(seed + 500_000).standard_normal((m, n))


# ---------------------------------------------------------------------------
# GPU generators (torch, float32): for large sets only, harness side
# ---------------------------------------------------------------------------

def _torch_haar(torch, gen, n: int, k: int, device):
    q, r = torch.linalg.qr(torch.randn(n, k, generator=gen, device=device, dtype=torch.float32))
    return q * torch.sign(torch.diagonal(r)).unsqueeze(0)


def gradient_gpu(config: int, m: int, n: int, seed: int, device, dtype):
    """Same recipe as gradient_cpu, generated on the device in float32."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    s = min(m, n)
    if config == CONFIG_MOE:
        sigma = log_spaced(s)
        noise = 0.0
    elif config == CONFIG_SWEEP:
        sigma = log_uniform(np.random.default_rng(seed + 7), s)
        noise = 0.0
    else:
        k = {CONFIG_SINGLE: s, CONFIG_GPT2: min(64, s), CONFIG_LLAMA: min(512, s)}[config]
        sigma = power_law(k)
        noise = 1e-3
    k = len(sigma)
    U = _torch_haar(torch, gen, m, k, device)
    V = _torch_haar(torch, gen, n, k, device)
    sig = torch.tensor(np.ascontiguousarray(sigma), dtype=torch.float32, device=device)
    G = (U * sig) @ V.T
    if noise:
        G += noise * torch.randn(m, n, generator=gen, device=device, dtype=torch.float32)
    return G.to(dtype)


def param_gpu(m: int, n: int, seed: int, device, std: float = 0.02):
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(seed + 500_000)
    return std * torch.randn(m, n, generator=gen, device=device, dtype=torch.float32)


# ---------------------------------------------------------------------------
# Values as the device holds them, and the input recipes of the parity tests
# ---------------------------------------------------------------------------

def as_float32_values(x):
    """float64 array holding the float32 values the device receives."""
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def as_bf16_values(x):
    """float64 array holding the bf16 values the device receives (a float32
    cast, then torch's cast to bfloat16, as the tests upload them)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(np.asarray(x, dtype=np.float32)))
    return t.to(torch.bfloat16).to(torch.float64).numpy()


def set_values(config: int, shapes, grad_bf16: bool, seed_base: int = 0, indices=None):
    """The parity tests' inputs for a shape set: {index: (p, g, m0)} with the
    values the device holds (float32 p, float32 or bf16 g, zero m0). Matrix
    i uses seed_for(config, i // 7, i % 7) + seed_base."""
    out = {}
    for i, (m, n) in enumerate(shapes):
        if indices is not None and i not in indices:
            continue
        seed = seed_for(config, i // 7, i % 7) + seed_base
        g = gradient_cpu(config, m, n, seed)
        g = as_bf16_values(g) if grad_bf16 else as_float32_values(g)
        out[i] = (as_float32_values(param_cpu(m, n, seed)), g, np.zeros((m, n)))
    return out


def gaussian_set(shapes, seed: int, scale: float = 1.0):
    """Standard-normal matrices (times scale) from one generator, in order,
    as bf16 values: the stage tests' inputs."""
    rng = np.random.default_rng(seed)
    return [as_bf16_values(rng.standard_normal((m, n)) * scale) for (m, n) in shapes]


def sweep_matrix(m: int, n: int, index: int):
    """bf16 values of NS-only sweep input `index` of an m x n point."""
    return as_bf16_values(gradient_cpu(CONFIG_SWEEP, m, n, seed_for(CONFIG_SWEEP, m // 128, n // 128, index)))


# Shape lists of the parity tests (one definition for the tests and for the
# script that freezes the bf16 program's errors on the same inputs).
PARITY_SHAPES = {
    # ragged tiles: 1 x 1, thin rows and columns, tails of 1, tall and wide
    "ragged": [(1, 1), (3, 5), (5, 3), (1, 300), (300, 1), (127, 129), (129, 127), (64, 64), (256, 512),
               (512, 256), (384, 384), (200, 1000), (1000, 200), (520, 520), (768, 2304)],
    # every matrix on the on-chip small path (s <= 128, l <= 512)
    "small": [(1, 1), (3, 5), (5, 3), (64, 64), (100, 300), (300, 100), (128, 128), (128, 512), (512, 128),
              (127, 129), (1, 300), (300, 1), (16, 512), (512, 16), (96, 200), (65, 65)],
    # NS-only sweep points (m, n, batch) small enough for the oracle
    "sweep": [(128, 128, 4), (128, 512, 2), (512, 128, 2), (256, 256, 3), (256, 2048, 1), (2048, 256, 1),
              (1024, 1024, 1), (512, 4096, 1)],
    "mixed": [(128, 512), (512, 128), (64, 64), (768, 768), (300, 100), (1024, 256), (2, 2)],
    "gram": [(256, 1024), (1024, 256), (384, 384), (300, 1000), (1000, 300), (600, 257), (128, 512), (64, 96)],
    "deterministic": [(2304, 768), (768, 3072), (300, 1000), (64, 96), (4096, 1024)],
    "split": [(2304, 768), (768, 768), (768, 3072)],
    "schedule": [(256, 768), (768, 256), (100, 300), (512, 512)],
    "wait": [(512, 1024), (1024, 512)],
    "layerwise": [(256, 768), (768, 256), (64, 64), (1024, 512), (512, 1024), (300, 700)],
    "noalloc": [(300, 700), (700, 300), (256, 256), (5, 3), (1024, 1024)],
    # extreme aspect ratios on the tiled phases: one K-block Grams of a
    # million-long row, million-row combines, a ragged 70001-long row
    "extreme": [(1, 1 << 20), (1 << 20, 1), (8, 131072), (131072, 8), (3, 70001)],
}

# Row blocks of the split-Muon test (None: the matrix stays whole).
SPLIT_ROWS = [768, 64, None]

# The varying coefficient table of the schedule test.
SCHEDULE_TABLE = [(3.4445, -4.7750, 2.0315), (3.0, -3.2, 1.2), (2.5, -2.0, 0.6), (1.875, -1.25, 0.375)]

# Sampled matrices of the full-size sets: Llama layer 0 q (square), k (wide,
# small), gate (tall) and layer 31 down (wide); three MoE experts' matrices.
LLAMA_SAMPLE = [0, 1, 4, 223]
MOE_SAMPLE = [0, 5, 382]


def case_key(x, steps: int, coeffs, normalised: bool) -> str:
    """Identity of one Newton-Schulz input: a digest of its float64 bytes,
    the iteration count, the coefficients and whether it is normalised."""
    import hashlib
    h = hashlib.sha256(np.ascontiguousarray(np.asarray(x, dtype=np.float64)).tobytes())
    h.update(repr((int(steps), [float(v) for v in np.ravel(coeffs)], bool(normalised))).encode())
    return h.hexdigest()[:20]


def ns_flops(m: int, n: int, steps: int = 5) -> float:
    """Nominal FLOPs of the Newton-Schulz phases: steps * (4 s^2 l + 2 s^3)."""
    s, l = min(m, n), max(m, n)
    return steps * (4.0 * s * s * l + 2.0 * s ** 3)


def gram_ns_flops(m: int, n: int, steps: int = 5) -> float:
    """Nominal FLOPs of the Gram form in segments of two steps: per
    two-step segment one Gram and one final product (2 s^2 l each) and five
    s x s products (2 s^3 each); a one-step segment is the plain step."""
    s, l = min(m, n), max(m, n)
    two, one = steps // 2, steps % 2
    return two * (4.0 * s * s * l + 10.0 * s ** 3) + one * (4.0 * s * s * l + 2.0 * s ** 3)


def ns_flops_symmetric(m: int, n: int, steps: int = 5) -> float:
    """The method's own work per matrix: the Gram and the polynomial are
    symmetric, so only their upper triangles are computed (s^2 l + s^3),
    plus the combine (2 s^2 l): steps * (3 s^2 l + s^3)."""
    s, l = min(m, n), max(m, n)
    return steps * (3.0 * s * s * l + 1.0 * s ** 3)


def gram_ns_flops_symmetric(m: int, n: int, steps: int = 5) -> float:
    """The Gram form's own work: per two-step segment one symmetric Gram
    (s^2 l), five symmetric s x s products (s^3 each) and the final product
    (2 s^2 l); a one-step segment is the plain step."""
    s, l = min(m, n), max(m, n)
    two, one = steps // 2, steps % 2
    return two * (3.0 * s * s * l + 5.0 * s ** 3) + one * (3.0 * s * s * l + 1.0 * s ** 3)


def total_ns_flops_symmetric(shapes, steps: int = 5, gram: bool = False) -> float:
    f = gram_ns_flops_symmetric if gram else ns_flops_symmetric
    return float(sum(f(m, n, steps) for m, n in shapes))


def shape_classes(shapes):
    """{(m, n): (count, first index)} of a shape set, in first-seen order."""
    out = {}
    for i, s in enumerate(shapes):
        s = (int(s[0]), int(s[1]))
        c, first = out.get(s, (0, i))
        out[s] = (c + 1, first)
    return out


def step_bytes(m: int, n: int, grad_bytes: int) -> tuple:
    """Algorithmic HBM bytes of the two elementwise kernels per matrix.

    momentum/norm/cast: read g and m, write m and the bf16 cast;
    apply: read p and the bf16 result, write p.
    """
    e = m * n
    return e * (grad_bytes + 4 + 4 + 2), e * (4 + 2 + 4)


def describe(config: int) -> str:
    return {
        CONFIG_SINGLE: "one 256x512 fp32 gradient, power-law spectrum i^-1.5 + 1e-3 noise",
        CONFIG_GPT2: "GPT-2-small hidden matrices (48), fp32 grads, rank-64 power law + 1e-3 noise",
        CONFIG_LLAMA: "Llama-3-8B hidden matrices (224), bf16 grads, power law i^-1.5 (cut at rank 512) + 1e-3 noise",
        CONFIG_MOE: "MoE layer, 128 experts x 3 matrices (384), bf16 grads, log-spaced spectrum, condition 1e4",
        CONFIG_SWEEP: "NS-only sweep, bf16 X, log-uniform singular values in [1e-4, 1]",
    }[config]


def total_elements(shapes) -> int:
    return int(sum(m * n for m, n in shapes))


def total_ns_flops(shapes, steps: int = 5, gram: bool = False) -> float:
    f = gram_ns_flops if gram else ns_flops
    return float(sum(f(m, n, steps) for m, n in shapes))


__all__ = [name for name in dir() if not name.startswith("_") and name not in ("annotations", "math", "np")]
