"""The allocation-free Newton-Schulz entry point (muon_newton_schulz_noalloc).

Some callers cannot allocate device memory when they run the stage (a stream
captured in global mode, a fixed-budget pool allocator that owns all device
memory, a latency-critical path): this entry point keeps all its scratch in a
static device array instead. Here it is called through the C ABI and its
output is compared with the handle-based entry point (muon_newton_schulz) on
the same inputs, for two calls in a row; an oversized shape table must be
rejected with a clear message. Collected last so that a failure here never
hides the other tests; it also passes alone in a fresh process.
"""

import ctypes

import numpy as np
import pytest
import torch

import muon_newton_schulz_03_b200 as muon

from gpu_helpers import DEV, TOL_BF16_EMU, rel, to64, x_buffer

pytestmark = pytest.mark.gpu


def _arrays(xs):
    arr = (ctypes.c_void_p * len(xs))()
    for i, x in enumerate(xs):
        arr[i] = x.data_ptr()
    return arr


def _shapes(shapes):
    arr = (ctypes.c_int32 * (3 * len(shapes)))()
    for i, (m, n) in enumerate(shapes):
        arr[3 * i], arr[3 * i + 1], arr[3 * i + 2] = m, n, 0
    return arr


def _noalloc(xin, xout, shapes, sumsq, steps, err):
    lib = muon.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.muon_newton_schulz_noalloc(_arrays(xin), _arrays(xout),
                                          None if sumsq is None else sumsq.data_ptr(), _shapes(shapes),
                                          len(shapes), steps, None, err.data_ptr(), stream)


@pytest.mark.parametrize("seed", [0])
def test_noalloc_matches_handle_entry_point_twice(seed):
    shapes = [(300, 700), (700, 300), (256, 256), (5, 3), (1024, 1024)]
    opt = muon.Muon(device=0)
    err = torch.full((1,), -1, dtype=torch.int32, device=DEV)
    for call in range(2):   # two calls in a row, fresh inputs each time
        rng = np.random.default_rng(seed + call)
        xin = [x_buffer(m, n, fill=rng.standard_normal((m, n))) for (m, n) in shapes]
        sumsq = torch.tensor([float(torch.sum(x[:, :n].double() ** 2)) for x, (m, n) in zip(xin, shapes)],
                             dtype=torch.float64, device=DEV)
        ref = [x_buffer(m, n) for (m, n) in shapes]
        got = [x_buffer(m, n) for (m, n) in shapes]
        opt.newton_schulz(xin, ref, shapes, sumsq, ns_steps=5)
        rc = _noalloc(xin, got, shapes, sumsq, 5, err)
        assert rc == 0, muon.load().muon_last_error()
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        for i, (m, n) in enumerate(shapes):
            a, b = to64(got[i][:, :n]), to64(ref[i][:, :n])
            assert rel(a, b) <= TOL_BF16_EMU, f"call {call} matrix {i}: {rel(a, b):.3e}"
    opt.close()


def test_noalloc_rejects_oversized_scratch():
    lib = muon.load()
    shapes = [(4096, 4096)]   # the X ping-pong buffers alone need 64 MiB
    xin = [x_buffer(4096, 4096)]
    xout = [x_buffer(4096, 4096)]
    err = torch.zeros((1,), dtype=torch.int32, device=DEV)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.muon_newton_schulz_noalloc(_arrays(xin), _arrays(xout), None, _shapes(shapes), 1, 5,
                                        None, err.data_ptr(), stream)
    assert rc == 1   # MUON_ERR_INVALID_ARG
    msg = lib.muon_last_error().decode()
    assert "scratch" in msg and str(64 * 1024 * 1024) in msg
