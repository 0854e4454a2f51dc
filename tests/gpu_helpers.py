"""Helpers shared by the GPU parity tests (inputs, comparisons)."""

import numpy as np
import torch

import muon_newton_schulz_03_b200 as muon
import workloads as W

DEV = torch.device("cuda:0")

# Tolerances (relative Frobenius unless stated), from the stated gates:
TOL_BF16_NS = 2e-2      # bf16 Newton-Schulz vs the float64 oracle
TOL_FP32_NS = 1e-4      # fp32 debug Newton-Schulz vs the float64 oracle
TOL_ELEM = 1e-6         # elementwise stages vs the float64 oracle
TOL_BF16_EMU = 1e-2     # bf16 Newton-Schulz vs the oracle's bf16-rounding mode


def bf16_gate(got, exact, emulated, emulated32, what=""):
    """Two-tier parity of a bf16 Newton-Schulz result.

    `emulated` and `emulated32` are the oracle at the pages' precision (bf16
    rounding of the input and of every Gram / polynomial / combine output),
    accumulating in float64 and in float32: two equally valid bf16
    realizations. Their distance, `spread`, measures how strongly rounding
    differences grow through the iteration at this input (tiny for
    well-conditioned inputs, ~1e-2 and more when singular values reach down to
    1e-4 without normalisation).
    1. The GPU is a bf16 realization: its distance to the nearer of the two
       is within max(TOL_BF16_EMU, 3 * spread, inherent / 2). The last term
       only matters where bf16 arithmetic is far from exact (inherent above
       the gate): there the tensor cores' accumulation makes a third
       realization whose drift the float32 emulation does not bound.
    2. The GPU is as accurate as bf16 arithmetic allows: its distance to the
       exact float64 oracle is within TOL_BF16_NS, or, where bf16 arithmetic
       itself cannot meet that (the emulations' own distance `inherent`
       exceeds it), within 1.05 * inherent + 3 * spread.
    Returns (err_vs_exact, err_vs_emulated, inherent, spread).
    """
    e_emu = min(rel(got, emulated), rel(got, emulated32))
    e_exact = rel(got, exact)
    inherent = max(rel(emulated, exact), rel(emulated32, exact))
    spread = rel(emulated32, emulated)
    bound1 = max(TOL_BF16_EMU, 3.0 * spread, 0.5 * inherent if inherent > TOL_BF16_NS else 0.0)
    assert e_emu <= bound1, f"{what}: {e_emu:.3e} from the bf16-rounding oracle (spread {spread:.3e})"
    bound2 = TOL_BF16_NS if inherent <= TOL_BF16_NS else 1.05 * inherent + 3.0 * spread
    assert e_exact <= bound2, (f"{what}: {e_exact:.3e} from the exact oracle "
                               f"(bf16 arithmetic alone: {inherent:.3e}, spread {spread:.3e})")
    return e_exact, e_emu, inherent, spread


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
    """CPU-generated inputs: list of (p, g, m) float64 arrays and torch CUDA tensors."""
    cpu, dev = [], []
    for i, (m, n) in enumerate(shapes):
        seed = W.seed_for(config, i // 7, i % 7) + seed_base
        g = W.gradient_cpu(config, m, n, seed)
        p = W.param_cpu(m, n, seed)
        mom = np.zeros((m, n))
        gt = (cuda_bf16(g) if grad_dtype == torch.bfloat16 else cuda_f32(g))
        pt, mt = cuda_f32(p), cuda_f32(mom)
        cpu.append((to64(pt), to64(gt), to64(mt)))
        dev.append((pt, gt, mt))
    return cpu, dev


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
