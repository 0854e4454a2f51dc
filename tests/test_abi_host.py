"""Host-side checks of the C ABI (no GPU needed).

* the shared library builds, loads and exports every function that
  include/muon_ns.h declares;
* the integer plan tables match the independent restatement in
  oracle/plan_tables.py bit for bit, for the workload shape sets and for
  ragged shapes;
* the tile lists cover every output entry exactly once (brute force);
* invalid arguments are rejected with MUON_ERR_INVALID_ARG, and a missing
  GPU is reported, not crashed on.
"""

import os
import re

import numpy as np
import pytest

import muon_newton_schulz_03_b200 as muon
from muon_newton_schulz_03_b200 import _lib
from oracle import plan_tables as PT
import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(muon_[a-z_0-9]+)\s*\(", text))
    return names


def test_library_exports_every_declared_function():
    lib = muon.load()
    declared = _declared_functions()
    assert len(declared) >= 15
    for name in declared:
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"
    assert declared == set(_lib.EXPORTED)
    assert b"sm_100a" in lib.muon_version()


SHAPE_SETS = {
    "single": W.single_shapes(),
    "gpt2": W.gpt2_shapes(),
    "llama3": W.llama3_8b_shapes(),
    "moe": W.moe_shapes(),
    "ragged": [(1, 1), (1, 7), (7, 1), (3, 5), (127, 129), (129, 127), (300, 300), (513, 257), (64, 1000),
               (1000, 64), (256, 256), (255, 257)],
}


@pytest.mark.parametrize("name", sorted(SHAPE_SETS))
@pytest.mark.parametrize("prec", ["bf16", "fp32"])
@pytest.mark.parametrize("small_path", [True, False])
@pytest.mark.parametrize("pair", [True, False])
def test_plan_tables_bit_exact(name, prec, small_path, pair):
    shapes = SHAPE_SETS[name]
    got = muon.plan_query(shapes, prec, small_path, pair)
    regions, ws, _ = PT.workspace_layout(shapes, 2 if prec == "bf16" else 4)
    assert got["ws_bytes"] == ws
    assert got["region_offsets"] == regions
    gram, poly, comb, small = PT.tile_lists(shapes, small_path, pair)
    assert got["tiles"][0] == gram
    assert got["tiles"][1] == poly
    assert got["tiles"][2] == comb
    assert got["small"] == small
    assert got["chunk_prefix"] == PT.chunk_prefix(shapes)


@pytest.mark.parametrize("shape", [(1, 1), (5, 3), (130, 300), (300, 130), (512, 512), (600, 257), (257, 600),
                                   (1000, 700)])
@pytest.mark.parametrize("pair", [False, True])
def test_tiles_cover_each_entry_once(shape, pair):
    m, n = shape
    bm = PT.BM_PAIR if pair else PT.BM
    got = muon.plan_query([shape], small_path=False, cta_pair=pair)
    s = min(m, n)
    # Symmetric phases: direct writes of each listed tile plus transposed
    # writes of the tiles whose column block starts after their row block.
    for tiles in got["tiles"][:2]:
        cover = np.zeros((s, s), dtype=np.int64)
        for (_, ti, tj) in tiles:
            r0, c0 = ti * bm, tj * PT.BN
            r1, c1 = min(r0 + bm, s), min(c0 + PT.BN, s)
            cover[r0:r1, c0:c1] += 1
            if PT.mirrored(ti, tj, bm):
                cover[c0:c1, r0:r1] += 1
        assert np.all(cover == 1)
    cover = np.zeros((m, n), dtype=np.int64)
    for (_, ti, tj) in got["tiles"][2]:
        cover[ti * bm:(ti + 1) * bm, tj * PT.BN:(tj + 1) * PT.BN] += 1
    assert np.all(cover == 1)


def test_workspace_regions_aligned_and_disjoint():
    shapes = SHAPE_SETS["ragged"]
    got = muon.plan_query(shapes)
    spans = []
    for (m, n), offs in zip(shapes, got["region_offsets"]):
        s = min(m, n)
        sizes = [m * muon.round_up(n, 8) * 2] * 2 + [s * muon.round_up(s, 8) * 2] * 2
        for o, sz in zip(offs, sizes):
            assert o % 1024 == 0
            spans.append((o, o + sz))
    spans.sort()
    assert spans[0][0] >= 8 * len(shapes)
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 <= b0
    assert spans[-1][1] <= got["ws_bytes"]


@pytest.mark.parametrize("bad", [[(0, 4)], [(4, 0)], [(-1, 4)], [(4, 1 << 21)], [(4, 4, 2)]])
def test_plan_rejects_invalid_shapes(bad):
    with pytest.raises(muon.MuonError) as e:
        muon.plan_query(bad)
    assert e.value.code == 1


def test_plan_rejects_empty_and_bad_precision():
    lib = muon.load()
    import ctypes
    arr = (ctypes.c_int32 * 3)(4, 4, 0)
    assert lib.muon_plan_query(arr, 0, 0, 1, None, None, None, None, None) == 1
    assert lib.muon_plan_query(arr, 1, 7, 1, None, None, None, None, None) == 1
    assert lib.muon_plan_query(None, 1, 0, 1, None, None, None, None, None) == 1
    assert b"shapes" in lib.muon_last_error()
    assert lib.muon_plan_query(arr, 1, 0, 8, None, None, None, None, None) == 1
    assert b"flags" in lib.muon_last_error()


def test_config_defaults():
    cfg = _lib.MuonConfig()
    lib = muon.load()
    import ctypes
    assert lib.muon_config_init(ctypes.byref(cfg)) == 0
    assert cfg.scale_mode == 0 and cfg.extra_scale == 1.0 and cfg.ns_precision == 0
    assert cfg.wait_timeout_s == 2.0 and cfg.num_sms == 0 and cfg.small_path == 1 and cfg.cta_pair == 0
    assert cfg.ns_algorithm == 0 and cfg.deterministic == 0
    assert lib.muon_config_init(None) == 1


def test_init_without_gpu_reports_no_device():
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(muon.MuonError) as e:
        muon.Muon(device=0)
    assert e.value.code == 6


def test_null_handle_rejected():
    lib = muon.load()
    assert lib.muon_step(None, None, None, None, None, 1, 0.1, 0.9, 1, 0.0, 5, None, None) == 1
    assert lib.muon_destroy(None) == 0


@pytest.mark.parametrize("field,value", [("ns_algorithm", 2), ("deterministic", 2)])
def test_init_rejects_bad_config_values(field, value):
    lib = muon.load()
    import ctypes
    cfg = _lib.MuonConfig()
    assert lib.muon_config_init(ctypes.byref(cfg)) == 0
    setattr(cfg, field, value)
    h = ctypes.c_void_p()
    assert lib.muon_init(0, ctypes.byref(cfg), ctypes.byref(h)) == 1
    assert field.encode() in lib.muon_last_error()


@pytest.mark.parametrize("other", [("ns_precision", 1), ("cta_pair", 1)])
def test_gram_form_needs_bf16_single_cta(other):
    # Checked before any device is touched, so it runs without a GPU.
    lib = muon.load()
    import ctypes
    cfg = _lib.MuonConfig()
    lib.muon_config_init(ctypes.byref(cfg))
    cfg.ns_algorithm = 1
    setattr(cfg, other[0], other[1])
    h = ctypes.c_void_p()
    assert lib.muon_init(0, ctypes.byref(cfg), ctypes.byref(h)) == 1
    assert b"Gram" in lib.muon_last_error()


@pytest.mark.parametrize("name", ["gpt2", "llama3", "moe", "ragged"])
@pytest.mark.parametrize("frac", [1.0, 0.5, 0.23, 0.05])
def test_capped_plan_groups_bit_exact(name, frac):
    # Under a workspace cap the matrices are packed into consecutive groups
    # that share one workspace; the C++ plan and the restatement agree.
    shapes = SHAPE_SETS[name]
    _, full, _ = PT.workspace_layout(shapes)
    cap = int(full * frac)
    try:
        regions, ws, bounds = PT.workspace_layout(shapes, 2, cap)
    except ValueError:
        with pytest.raises(muon.MuonError) as e:
            muon.plan_groups(shapes, cap)
        assert e.value.code == 3
        return
    got = muon.plan_groups(shapes, cap)
    assert got["bounds"] == bounds and got["region_offsets"] == regions and got["ws_bytes"] == ws
    assert ws <= cap
    if frac == 1.0:
        assert bounds == [0, len(shapes)] and got["region_offsets"] == muon.plan_query(shapes)["region_offsets"]
    # Regions of one group are aligned and disjoint.
    for g0, g1 in zip(bounds[:-1], bounds[1:]):
        spans = []
        for i in range(g0, g1):
            m, n = shapes[i]
            s = min(m, n)
            sizes = [m * muon.round_up(n, 8) * 2] * 2 + [s * muon.round_up(s, 8) * 2] * 2
            spans += [(o, o + z) for o, z in zip(got["region_offsets"][i], sizes)]
        spans.sort()
        assert all(a1 <= b0 for (_, a1), (b0, _) in zip(spans, spans[1:]))
        assert spans[-1][1] <= ws


def test_capped_plan_rejects_a_matrix_above_the_cap():
    with pytest.raises(muon.MuonError) as e:
        muon.plan_groups([(4096, 4096), (64, 64)], 1 << 20)
    assert e.value.code == 3 and "matrix 0" in str(e.value)
