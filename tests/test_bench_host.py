"""Host-side checks of the benchmark's FLOP and byte accounting (no GPU)."""

import pytest

import bench
import workloads as W


def test_nominal_flops_formula():
    # 4 s^2 l + 2 s^3 per iteration, s = min, l = max; orientation-free.
    assert W.ns_flops(256, 512, 1) == 4 * 256 ** 2 * 512 + 2 * 256 ** 3
    assert W.ns_flops(512, 256, 5) == W.ns_flops(256, 512, 5) == 5 * (4 * 256 ** 2 * 512 + 2 * 256 ** 3)


def test_gram_form_flops_formula():
    # Two-step segment: Gram + final product (2 s^2 l each) + five s^3 products.
    s, l = 1024, 4096
    assert W.gram_ns_flops(s, l, 2) == 4 * s * s * l + 10 * s ** 3
    assert W.gram_ns_flops(s, l, 1) == W.ns_flops(s, l, 1)
    assert W.gram_ns_flops(l, s, 5) == 2 * (4 * s * s * l + 10 * s ** 3) + W.ns_flops(s, l, 1)


def test_executed_flops_hand_count():
    # 512 x 1024 (wide, s = 512, l = 1024): Gram upper tiles with 128-row and
    # 256-column tiles are (ti, tj) with tj >= ti // 2: tj = 0 -> ti 0, 1;
    # tj = 1 -> ti 0..3 (4 row tiles of 128): 6 tiles; the polynomial lists the
    # same 6; the combine covers 512 x 1024 with 4 x 4 = 16 tiles.
    per_tile = 2 * 128 * 256
    gram = 6 * per_tile * 1024
    poly = 6 * per_tile * 512
    comb = 16 * per_tile * 512
    assert bench.executed_flops([(512, 1024)], 1) == gram + poly + comb
    assert bench.executed_flops([(512, 1024)], 5) == 5 * (gram + poly + comb)
    # Gram form, two steps: Gram + 5 symmetric products + combine.
    assert bench.executed_flops([(512, 1024)], 2, gram=True) == gram + 5 * poly + comb


def test_executed_flops_small_path_counts_nominal():
    # 128 x 128 runs on the on-chip path: counted at its nominal FLOPs.
    assert bench.executed_flops([(128, 128)], 5) == W.ns_flops(128, 128, 5)


@pytest.mark.parametrize("name", ["llama3", "gpt2", "moe"])
def test_executed_below_nominal_for_tiled_sets(name):
    shapes = {"llama3": W.llama3_8b_shapes(), "gpt2": W.gpt2_shapes(), "moe": W.moe_shapes()}[name]
    ratio = bench.executed_flops(shapes, 5) / W.total_ns_flops(shapes, 5)
    # Symmetric upper tiles save part of the Gram and polynomial work.
    assert 0.6 < ratio < 0.9


def test_elementwise_bytes():
    # K1: g + m read, m + bf16 X written; K4: p + bf16 O read, p written.
    assert W.step_bytes(10, 10, 2) == (100 * 12, 100 * 10)
    assert W.step_bytes(10, 10, 4) == (100 * 14, 100 * 10)


def test_executed_flops_pair_tiles_hand_count():
    # 256 x 256 tiles on CTA pairs, 512 x 1024: upper tiles (0,0), (0,1), (1,1)
    # for the symmetric phases, 2 x 4 = 8 combine tiles.
    per_tile = 2 * 256 * 256
    want = 3 * per_tile * 1024 + 3 * per_tile * 512 + 8 * per_tile * 512
    assert bench.executed_flops([(512, 1024)], 1, pair=True) == want


def test_symmetric_flops_formula():
    # Upper triangles of the Gram (s^2 l) and polynomial (s^3), full combine
    # (2 s^2 l): 3 s^2 l + s^3 per iteration, between the executed tile count
    # and the nominal dense count on the tiled sets.
    s, l = 256, 512
    assert W.ns_flops_symmetric(s, l, 1) == 3 * s * s * l + s ** 3
    assert W.ns_flops_symmetric(l, s, 5) == 5 * (3 * s * s * l + s ** 3)
    assert W.gram_ns_flops_symmetric(s, l, 2) == 3 * s * s * l + 5 * s ** 3
    assert W.gram_ns_flops_symmetric(s, l, 5) == 2 * (3 * s * s * l + 5 * s ** 3) + W.ns_flops_symmetric(s, l, 1)
    shapes = W.llama3_8b_shapes()
    alg = W.total_ns_flops_symmetric(shapes)
    assert alg < bench.executed_flops(shapes, 5) < W.total_ns_flops(shapes)
    assert abs(alg / 1e12 - 471.8) < 0.5     # TFLOP per Muon step on the Llama-3-8B set


def test_shape_classes_and_set_extrapolation():
    classes = W.shape_classes(W.llama3_8b_shapes())
    assert classes == {(4096, 4096): (64, 0), (1024, 4096): (64, 1), (14336, 4096): (64, 4), (4096, 14336): (32, 6)}
    secs = {(4096, 4096): 1.0, (1024, 4096): 0.5, (14336, 4096): 2.0, (4096, 14336): 3.0}
    assert bench.set_seconds("llama3", secs) == 64 * 1.0 + 64 * 0.5 + 64 * 2.0 + 32 * 3.0
    assert W.shape_classes(W.moe_shapes()) == {(2048, 7168): (256, 0), (7168, 2048): (128, 2)}


def test_tensor_peak_follows_the_length_of_the_timed_region():
    # A timed region of a second or more runs at the power cap: the sustained
    # figure; a shorter one at full clock: the burst figure.
    peaks = dict(bench.FALLBACK)
    tf, note = bench.tensor_peak(peaks, "fallback", 4300.0)
    assert tf == peaks["bf16_tflops_sustained"] and "sustained" in note and "4.3 s" in note
    tf, note = bench.tensor_peak(peaks, "fallback", 15.0)
    assert tf == peaks["bf16_tflops"] and "burst" in note and "15 ms" in note
    assert bench.tensor_peak(peaks, "measured", 1000.0)[0] == peaks["bf16_tflops_sustained"]
