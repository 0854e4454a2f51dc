"""The Python binding's argument marshalling (no GPU): the checks that the C
side cannot make (tensor sizes, dtypes, devices) and the arrays it builds."""

import ctypes

import pytest
import torch

import muon_newton_schulz_03_b200 as muon
from muon_newton_schulz_03_b200 import _marshal_step


def _set(shapes, gdtype=torch.float32):
    P = [torch.zeros(s) for s in shapes]
    G = [torch.zeros(s, dtype=gdtype) for s in shapes]
    M = [torch.zeros(s) for s in shapes]
    return P, G, M


def test_arrays_and_shape_table():
    shapes = [(3, 5), (7, 2), (1, 1)]
    P, G, M = _set(shapes)
    G[1] = G[1].to(torch.bfloat16)
    G[2] = None
    pa, ga, ma, sa, n = _marshal_step(P, G, M, host=True)
    assert n == 3
    assert list(sa) == [3, 5, 0, 7, 2, muon.FLAG_GRAD_BF16, 1, 1, 0]
    assert [pa[i] for i in range(3)] == [t.data_ptr() for t in P]
    assert [ma[i] for i in range(3)] == [t.data_ptr() for t in M]
    assert ga[0] == G[0].data_ptr() and ga[1] == G[1].data_ptr() and ga[2] is None
    assert isinstance(pa, ctypes.Array) and isinstance(sa, ctypes.Array)


@pytest.mark.parametrize("bad,exc,msg", [
    ("grad_shape", ValueError, "grads[1] shape"),
    ("mom_shape", ValueError, "momenta[1] shape"),
    ("param_dtype", TypeError, "params[1] must have dtype"),
    ("grad_dtype", TypeError, "grads[1] must have dtype"),
    ("mom_dtype", TypeError, "momenta[1] must have dtype"),
    ("not_2d", ValueError, "params[1] must be 2D"),
    ("non_contiguous", ValueError, "params[1] must be contiguous"),
])
def test_rejections(bad, exc, msg):
    shapes = [(4, 6), (6, 4)]
    P, G, M = _set(shapes)
    if bad == "grad_shape":
        G[1] = torch.zeros(4, 6)
    elif bad == "mom_shape":
        M[1] = torch.zeros(6, 5)
    elif bad == "param_dtype":
        P[1] = P[1].double()
    elif bad == "grad_dtype":
        G[1] = G[1].half()
    elif bad == "mom_dtype":
        M[1] = M[1].to(torch.bfloat16)
    elif bad == "not_2d":
        P[1] = torch.zeros(24)
    elif bad == "non_contiguous":
        P[1] = torch.zeros(4, 6).t()
    with pytest.raises(exc) as e:
        _marshal_step(P, G, M, host=True)
    assert msg in str(e.value)


def test_device_side_must_not_be_host_memory():
    P, G, M = _set([(2, 2)])
    with pytest.raises(ValueError) as e:
        _marshal_step(P, G, M, host=False)
    assert "CUDA device" in str(e.value)


def test_length_mismatch():
    P, G, M = _set([(2, 2), (3, 3)])
    with pytest.raises(ValueError):
        _marshal_step(P, G[:1], M, host=True)
