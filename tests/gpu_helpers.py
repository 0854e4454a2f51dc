"""Helpers shared by the GPU parity tests (inputs, comparisons)."""

import json
import os

import numpy as np
import torch

import muon_newton_schulz_03_b200 as muon
import workloads as W
from oracle import muon_oracle as O

DEV = torch.device("cuda:0")

# Tolerances (relative Frobenius unless stated), from the stated gates:
TOL_BF16_NS = 2e-2      # bf16 Newton-Schulz vs the float64 oracle
TOL_FP32_NS = 1e-4      # fp32 debug Newton-Schulz vs the float64 oracle
TOL_ELEM = 1e-6         # elementwise stages vs the float64 oracle
TOL_GPU_VS_GPU = 1e-2   # two GPU kernels with the same rounding points (small path vs tiled phases)

_GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "bf16_program_errors.json")
_PROGRAM_ERRORS = None


def bf16_program_error(x, steps=5, coeffs=O.DEFAULT_COEFFS, normalised=True):
    """Frozen distance from exact of the pages' bf16 program on this input.

    The values were written once by tests/golden/make_bf16_program_errors.py
    (oracle only) and are looked up by a digest of the input's float64
    bytes, the step count, the coefficients and the normalisation flag; an
    input that is not in the file is an error, never a default.
    """
    global _PROGRAM_ERRORS
    if _PROGRAM_ERRORS is None:
        with open(_GOLDEN) as f:
            _PROGRAM_ERRORS = json.load(f)["cases"]
    key = W.case_key(x, steps, coeffs, normalised)
    if key not in _PROGRAM_ERRORS:
        raise KeyError(f"no frozen bf16-program distance for input {key}: "
                       "rerun tests/golden/make_bf16_program_errors.py")
    return _PROGRAM_ERRORS[key]["err"]


def bf16_ns_tolerance(x, steps=5, coeffs=O.DEFAULT_COEFFS, normalised=True):
    """The bf16 gate on a Newton-Schulz output: 2e-2 from exact, or the
    pages' own bf16 program's distance from exact where that is larger."""
    return max(TOL_BF16_NS, bf16_program_error(x, steps, coeffs, normalised))


def report(what, err, tol, program=None):
    """One line per gated comparison (shown with pytest -s)."""
    extra = "" if program is None else f" program={program:.3e}"
    print(f"PARITY {what}: gpu={err:.3e} gate={tol:.3e}{extra}")


def gate_bf16_ns(got, exact, x, steps=5, coeffs=O.DEFAULT_COEFFS, normalised=True, what=""):
    """Assert the bf16 gate on O; returns (error, tolerance)."""
    prog = bf16_program_error(x, steps, coeffs, normalised)
    tol = max(TOL_BF16_NS, prog)
    e = rel(got, exact)
    report(f"O {what}", e, tol, prog)
    assert e <= tol, f"{what}: {e:.3e} from the exact oracle (gate {tol:.3e})"
    return e, tol


def gate_bf16_update(p_gpu, p0, p_exact, o_exact, lr_scale, tol_o, what=""):
    """The same gate carried to the update dp = p' - p.

    p' = p (1 - lr wd) - lr scale O, so an error E in O moves dp by
    lr scale E: the O tolerance becomes tol_o * lr scale ||O|| / ||dp||,
    plus the float32 rounding of the written p' (2^-23 of ||p'||)."""
    dp_exact = p_exact - p0
    ndp = np.linalg.norm(dp_exact)
    tol = (tol_o * abs(lr_scale) * np.linalg.norm(o_exact) + 2.0 ** -23 * np.linalg.norm(p_exact)) / ndp
    e = rel(p_gpu - p0, dp_exact)
    report(f"dp {what}", e, tol)
    assert e <= tol, f"{what}: update {e:.3e} from the exact oracle (gate {tol:.3e})"
    return e


def rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (nb if nb > 0 else 1.0)


def to64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def cuda_f32(a):
    return torch.as_tensor(np.asarray(a), dtype=torch.float32).to(DEV)


def cuda_bf16(a):
    return torch.as_tensor(np.asarray(a), dtype=torch.float32).to(torch.bfloat16).to(DEV)


def x_buffer(m, n, dtype=torch.bfloat16, fill=None):
    buf = muon.x_layout(m, n, dtype, DEV)
    if fill is not None:
        buf.zero_()
        buf[:, :n] = torch.as_tensor(np.asarray(fill), dtype=torch.float32).to(dtype).to(DEV)
    return buf


def bf16_ulp(x):
    """Spacing of bf16 numbers at |x| (for normal values)."""
    ax = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, 2.0 ** (e - 7), 2.0 ** -133)


def make_set(config, shapes, grad_dtype, seed_base=0):
    """Inputs of a shape set (workloads.set_values): list of (p, g, m)
    float64 arrays holding the device's values, and the CUDA tensors."""
    vals = W.set_values(config, shapes, grad_dtype == torch.bfloat16, seed_base)
    cpu, dev = [], []
    for i in range(len(shapes)):
        p, g, mom = vals[i]
        gt = (cuda_bf16(g) if grad_dtype == torch.bfloat16 else cuda_f32(g))
        pt, mt = cuda_f32(p), cuda_f32(mom)
        cpu.append((to64(pt), to64(gt), to64(mt)))
        assert np.array_equal(cpu[-1][1], g)
        dev.append((pt, gt, mt))
    return cpu, dev


def gaussian_buffers(shapes, seed, scale=1.0, dtype=torch.bfloat16):
    """workloads.gaussian_set in the library's X layout: (buffers, float64 values)."""
    xs = W.gaussian_set(shapes, seed, scale)
    bufs = [x_buffer(m, n, dtype, fill=x) for (m, n), x in zip(shapes, xs)]
    vals = [to64(b[:, :n]) for b, (m, n) in zip(bufs, shapes)]
    for a, b in zip(vals, xs):
        assert np.array_equal(a, b)
    return bufs, vals


def workspace_matrix(opt, shapes, index, region, dtype=torch.bfloat16):
    """View of one workspace region (0: X0, 1: X1, 2: A, 3: B) of matrix `index`."""
    plan = muon.plan_query(shapes, opt.ns_precision)
    base, size = opt.workspace()
    off = plan["region_offsets"][index][region]
    m, n = shapes[index]
    s = min(m, n)
    rows, cols = (m, muon.round_up(n, 8)) if region < 2 else (s, muon.round_up(s, 8))
    esz = 2 if dtype == torch.bfloat16 else 4
    nbytes = rows * cols * esz
    assert off + nbytes <= size
    return device_view(base + off, (rows, cols), dtype).clone()


class _CudaArray:
    def __init__(self, ptr, shape, typestr):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr, "data": (int(ptr), False),
                                         "version": 3, "strides": None}


def device_view(ptr, shape, dtype):
    """A torch tensor aliasing raw device memory (bf16 or fp32)."""
    torch.cuda.synchronize()
    if dtype == torch.bfloat16:
        t = torch.as_tensor(_CudaArray(ptr, shape, "<i2"), device=DEV)
        return t.view(torch.bfloat16)
    return torch.as_tensor(_CudaArray(ptr, shape, "<f4"), device=DEV)
