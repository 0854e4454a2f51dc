"""The allocation-free Newton-Schulz entry point (muon_newton_schulz_noalloc).

Some callers cannot allocate device memory when they run the stage: a
process whose device memory belongs to its own fixed-budget pool allocator,
or a serving process that reserved its memory at start-up and must keep its
footprint fixed. This entry point keeps all its scratch in a static device
array instead. Here it is called through the C ABI, for two calls in a row
with fresh inputs, and compared with the float64 oracle (at the bf16 gate)
and with the handle-based entry point muon_newton_schulz on the same inputs;
ns_steps 0, 1 and 5 and the unnormalised form (sumsq = NULL) are covered. An
oversized shape table, a pointer that is not device memory and a call on a
stream that is being captured must be refused with a clear message.
Collected last so that a failure here never hides the other tests; it also
passes alone in a fresh process.
"""

import ctypes

import numpy as np
import pytest
import torch

import muon_newton_schulz_03_b200 as muon
import workloads as W
from oracle import muon_oracle as O

from gpu_helpers import DEV, TOL_GPU_VS_GPU, gate_bf16_ns, gaussian_buffers, rel, to64, x_buffer

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


def _noalloc(xin, xout, shapes, sumsq, steps, err, stream=None):
    lib = muon.load()
    st = torch.cuda.current_stream() if stream is None else stream
    return lib.muon_newton_schulz_noalloc(_arrays(xin), _arrays(xout),
                                          None if sumsq is None else sumsq.data_ptr(), _shapes(shapes),
                                          len(shapes), steps, None, err.data_ptr(), ctypes.c_void_p(st.cuda_stream))


@pytest.mark.parametrize("steps", [5, 1, 0])
def test_noalloc_matches_oracle_and_handle_entry_point_twice(steps):
    shapes = W.PARITY_SHAPES["noalloc"]
    opt = muon.Muon(device=0)
    err = torch.full((1,), -1, dtype=torch.int32, device=DEV)
    for call in range(2):   # two calls in a row, fresh inputs each time
        xin, x64 = gaussian_buffers(shapes, call)
        sumsq = torch.tensor([float(np.sum(x ** 2)) for x in x64], dtype=torch.float64, device=DEV)
        ref = [x_buffer(m, n) for (m, n) in shapes]
        got = [x_buffer(m, n) for (m, n) in shapes]
        opt.newton_schulz(xin, ref, shapes, sumsq, ns_steps=steps)
        rc = _noalloc(xin, got, shapes, sumsq, steps, err)
        assert rc == 0, muon.load().muon_last_error()
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        for i, (m, n) in enumerate(shapes):
            a, b = to64(got[i][:, :n]), to64(ref[i][:, :n])
            assert rel(a, b) <= TOL_GPU_VS_GPU, f"call {call} matrix {i}: {rel(a, b):.3e} from the handle path"
            exact = O.newton_schulz(x64[i], steps)
            if steps == 0:
                # bf16 cast and one scaling: two bf16 roundings at most
                assert rel(a, exact) <= 4e-3
            else:
                gate_bf16_ns(a, exact, x64[i], steps, what=f"call {call} matrix {i} {m}x{n}")
    opt.close()


def test_noalloc_without_norm_on_scaled_inputs():
    # sumsq = NULL: the iteration runs on X as given (singular values already
    # in [1e-4, 1], the NS-only inputs), against the oracle's NS-only form.
    m, n, batch = 256, 256, 3
    shapes = [(m, n)] * batch
    xs = [W.sweep_matrix(m, n, b) for b in range(batch)]
    xin = [x_buffer(m, n, fill=x) for x in xs]
    got = [x_buffer(m, n) for _ in shapes]
    err = torch.full((1,), -1, dtype=torch.int32, device=DEV)
    rc = _noalloc(xin, got, shapes, None, 5, err)
    assert rc == 0, muon.load().muon_last_error()
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for b in range(batch):
        gate_bf16_ns(to64(got[b][:, :n]), O.ns_only(xs[b], 5), xs[b], 5, normalised=False, what=f"#{b}")


def test_noalloc_rejects_oversized_scratch():
    lib = muon.load()
    shapes = [(4096, 4096)]   # the X ping-pong buffers alone need 64 MiB
    xin = [x_buffer(4096, 4096)]
    xout = [x_buffer(4096, 4096)]
    err = torch.zeros((1,), dtype=torch.int32, device=DEV)
    rc = _noalloc(xin, xout, shapes, None, 5, err)
    assert rc == 1   # MUON_ERR_INVALID_ARG
    msg = lib.muon_last_error().decode()
    assert "scratch" in msg and str(64 * 1024 * 1024) in msg


def test_noalloc_rejects_host_memory_and_capture():
    lib = muon.load()
    shapes = [(64, 96)]
    err = torch.zeros((1,), dtype=torch.int32, device=DEV)
    host = [torch.zeros(muon.x_layout(64, 96, torch.bfloat16, "cpu").shape, dtype=torch.bfloat16).pin_memory()]
    dev = [x_buffer(64, 96, fill=np.ones((64, 96)))]
    assert _noalloc(host, [x_buffer(64, 96)], shapes, None, 1, err) == 1
    assert "device memory" in lib.muon_last_error().decode()
    # A call on a stream being captured is refused before it enqueues
    # anything; the capture itself stays valid.
    out = [x_buffer(64, 96)]
    assert _noalloc(dev, out, shapes, None, 1, err) == 0       # set-up done outside capture
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    probe = torch.zeros(4, device=DEV)
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(graph, stream=side):
        probe.add_(1.0)
        rc = _noalloc(dev, out, shapes, None, 1, err, stream=side)
    assert rc == 1
    assert "captured" in lib.muon_last_error().decode()
    graph.replay()
    torch.cuda.synchronize()
    assert float(probe.sum()) == 4.0
    del graph
