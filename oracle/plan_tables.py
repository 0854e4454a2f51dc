"""Independent restatement of the integer plan tables (test infrastructure only).

Only ``tests/`` may import this module. The C++ plan builder in the CUDA
library produces the same tables; a test compares the two bit for bit.

The rules restated here:

Orientation ("About Muon: Why Not Adam", section "The whole thing, in about
forty lines"): a matrix with m > n (rows > columns) is "tall" and the
iteration runs on its transpose; s = min(m, n), l = max(m, n). Square
matrices are not transposed.

Storage. Every bf16 (or, in the fp32 debug mode, fp32) matrix in the
workspace is row-major with a leading dimension rounded up to a multiple of
8 elements, so each row starts on a 16-byte boundary (the alignment the
bulk-tensor copy engine requires):
  * X ping-pong buffers X0, X1: m rows, ldx = round_up(n, 8).
  * Gram A and polynomial B: s rows, lds = round_up(s, 8).
The workspace begins with one float64 sum-of-squares accumulator per
matrix, padded to 1024 bytes; then all X0 regions, all X1
regions, all A regions, all B regions, each region aligned to 1024 bytes.

Workspace cap. When that layout is larger than a cap, consecutive matrices
are packed into groups in index order, each group as large as fits under
the cap; every group lays out its own X0, X1, A and B regions (same order,
same alignment) starting right after the sum-of-squares block, so the
groups share one workspace and run one after another. A matrix whose
regions alone exceed the cap is rejected.

Tiles. Output tiles are BM rows by BN = 256 columns: BM = 128 on single
CTAs, BM = 256 on CTA pairs.
  * Gram and polynomial (both symmetric s x s): tile (ti, tj) is listed iff
    tj >= ti * BM // 256, i.e. its 256-wide column block is on or right of
    the 256-block diagonal. The entries of tiles whose column block starts
    at or after the end of their row block also stand for their mirror
    image (written transposed, or read transposed by the consumers), so each
    entry of the symmetric matrix is produced once.
  * Combine (output in the original m x n layout): every tile of the
    ceil(m/BM) x ceil(n/256) grid. For wide matrices (m <= n) the column
    block is the outer loop, for tall ones the row block.
  Each phase's list is ordered by the matrix's reduction length K
  (descending; Gram: K = l, polynomial and combine: K = s), ties by matrix
  index, then by the per-matrix order above. A tile entry is
  (matrix, ti, tj).

Small path. With the small path on (the default), a matrix with
s <= 128 and l <= 512 runs its whole iteration in one on-chip kernel: it is
left out of the three tile lists and listed, in matrix-index order, in a
fourth list.

Elementwise chunks. The fused momentum and apply kernels give each thread
block CHUNK = 8192 consecutive elements of one matrix; chunk_prefix[i] is
the number of chunks of matrices 0..i-1.
"""

from __future__ import annotations

BM = 128
BN = 256
CHUNK = 8192
ALIGN = 1024


def round_up(x: int, k: int) -> int:
    return (x + k - 1) // k * k


def ceil_div(x: int, k: int) -> int:
    return (x + k - 1) // k


def matrix_geometry(m: int, n: int):
    """(tall, s, l, ldx, lds) for an m x n matrix."""
    tall = m > n
    s = min(m, n)
    l = max(m, n)
    return tall, s, l, round_up(n, 8), round_up(s, 8)


def workspace_layout(shapes, elem_bytes: int = 2, cap: int = 0):
    """Byte offsets (X0, X1, A, B) per matrix, the workspace size and the
    group bounds (a list starting with 0 and ending with len(shapes))."""
    count = len(shapes)
    head = round_up(8 * count, ALIGN)

    def region(i, which):
        m, n = shapes[i]
        _, s, _, ldx, lds = matrix_geometry(m, n)
        return round_up((m * ldx if which < 2 else s * lds) * elem_bytes, ALIGN)

    sizes = [sum(region(i, w) for w in range(4)) for i in range(count)]
    bounds = [0]
    if cap and head + sum(sizes) > cap:
        used = 0
        for i, b in enumerate(sizes):
            if head + b > cap:
                raise ValueError(f"matrix {i} alone needs {head + b} bytes, above the cap {cap}")
            if head + used + b > cap:
                bounds.append(i)
                used = 0
            used += b
    bounds.append(count)
    regions = [[0, 0, 0, 0] for _ in range(count)]
    total = head
    for g0, g1 in zip(bounds[:-1], bounds[1:]):
        off = head
        for which in range(4):
            for i in range(g0, g1):
                regions[i][which] = off
                off += region(i, which)
        total = max(total, off)
    return regions, total, bounds


BM_PAIR = 256


def _sym_tiles(s: int, bm: int):
    out = []
    for ti in range(ceil_div(s, bm)):
        for tj in range(ti * bm // BN, ceil_div(s, BN)):
            out.append((ti, tj))
    return out


def mirrored(ti: int, tj: int, bm: int) -> bool:
    """Whether a symmetric tile also stands for its mirror image."""
    return tj * BN >= (ti + 1) * bm


def _comb_tiles(m: int, n: int, bm: int):
    rows, cols = ceil_div(m, bm), ceil_div(n, BN)
    if m <= n:   # wide: column block outer
        return [(ti, tj) for tj in range(cols) for ti in range(rows)]
    return [(ti, tj) for ti in range(rows) for tj in range(cols)]


SMALL_MAX_S = 128
SMALL_MAX_L = 512


def tile_lists(shapes, small_path=True, pair=False):
    """(gram, poly, comb) lists of (matrix, ti, tj) and the small-path list."""
    bm = BM_PAIR if pair else BM
    gram, poly, comb = [], [], []
    geo = [matrix_geometry(m, n) for (m, n) in shapes]
    small = [i for i, g in enumerate(geo) if small_path and g[1] <= SMALL_MAX_S and g[2] <= SMALL_MAX_L]
    tiled = set(range(len(shapes))) - set(small)

    def order(klen):
        return sorted(range(len(shapes)), key=lambda i: (-klen(i), i))

    for i in order(lambda i: geo[i][2]):
        if i in tiled:
            gram += [(i, ti, tj) for ti, tj in _sym_tiles(geo[i][1], bm)]
    for i in order(lambda i: geo[i][1]):
        if i in tiled:
            poly += [(i, ti, tj) for ti, tj in _sym_tiles(geo[i][1], bm)]
    for i in order(lambda i: geo[i][1]):
        if i in tiled:
            m, n = shapes[i]
            comb += [(i, ti, tj) for ti, tj in _comb_tiles(m, n, bm)]
    return gram, poly, comb, small


def chunk_prefix(shapes):
    out = [0]
    for (m, n) in shapes:
        out.append(out[-1] + ceil_div(m * n, CHUNK))
    return out
