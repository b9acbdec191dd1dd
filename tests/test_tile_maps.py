"""The grouped (mixture-of-experts) tile map of the tensor-core kernel (csrc/gemm_tc.cu: the
prologue's prefix sums and ``map_tile``), restated on the CPU and checked on random routings.

Per expert e with n_e routed rows: cum_m counts its pair (or single) tiles, 0 for an expert the
kernel skips (n_e <= skip_small: those run on the decode kernel with FS_PATH_DECODE), and cum_g
its 128-row groups in the packed activations (every expert padded to 128 rows, whether skipped or
not: the packed layout is fixed by the grouped quantiser).  Tile mt belongs to the last expert with
cum_m[e] <= mt; rank r of a CTA pair takes rows local * 128 CG + 128 r of the expert.

Checked: every row of every expert the kernel does not skip is written exactly once, by a CTA
whose packed A row is the same row of the expert's padded range; skipped and empty experts get no
rows; every CTA with rows reads scale atoms inside the packed buffer.
"""
import numpy as np
import pytest

KBM = 128


def prologue(counts, CG, skip_small):
    cum_m, cum_g = [0], [0]
    for n in counts:
        cum_m.append(cum_m[-1] + (0 if n <= skip_small else -(-n // (KBM * CG))))
        cum_g.append(cum_g[-1] + -(-n // KBM))
    return cum_m, cum_g


def map_tile(mt, rank, CG, offsets, cum_m, cum_g):
    E = len(offsets) - 1
    lo, hi = 0, E - 1
    while lo < hi:
        mid = (lo + hi + 1) >> 1
        if cum_m[mid] <= mt:
            lo = mid
        else:
            hi = mid - 1
    local = mt - cum_m[lo]
    off = local * (KBM * CG) + rank * KBM
    arow = cum_g[lo] * KBM + off
    yrow = offsets[lo] + off
    rows = min(offsets[lo + 1] - yrow, KBM)                 # <= 0: a pair's CTA past the expert
    return lo, arow, yrow, rows


def check(counts, CG, skip_small):
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64).tolist()
    cum_m, cum_g = prologue(counts, CG, skip_small)
    # the packed layout of the grouped quantiser: expert e's rows from pad[e], a 128-row boundary
    pad = np.concatenate([[0], np.cumsum([-(-n // KBM) * KBM for n in counts])]).astype(np.int64).tolist()
    written = np.zeros(offsets[-1], np.int64)
    for mt in range(cum_m[-1]):
        for rank in range(CG):
            e, arow, yrow, rows = map_tile(mt, rank, CG, offsets, cum_m, cum_g)
            assert counts[e] > skip_small, "a skipped or empty expert got a tile"
            if rows <= 0:
                continue
            assert offsets[e] <= yrow and yrow + rows <= offsets[e + 1]
            assert arow - pad[e] == yrow - offsets[e]               # the same row of the expert
            assert arow + rows <= pad[e + 1]                        # inside its padded range
            assert arow // KBM < pad[-1] // KBM                     # its scale atoms exist
            written[yrow:yrow + rows] += 1
    for e, n in enumerate(counts):
        want = 1 if n > skip_small else 0
        assert np.all(written[offsets[e]:offsets[e + 1]] == want), (e, n)


@pytest.mark.parametrize("CG", [1, 2])
@pytest.mark.parametrize("skip_small", [0, 16])
def test_grouped_tile_map_covers_every_row_once(CG, skip_small):
    rng = np.random.default_rng(100 * CG + skip_small)
    fixed = [[0], [1], [16], [17], [127, 128, 129, 255, 256, 257], [0, 0, 5, 0, 300, 0, 16, 17, 0]]
    for counts in fixed:
        check(counts, CG, skip_small)
    for _ in range(300):
        E = int(rng.integers(1, 65))
        kind = rng.integers(0, 3)
        if kind == 0:
            counts = rng.integers(0, 40, E)                          # decode-like: small experts
        elif kind == 1:
            counts = rng.integers(0, 700, E)                         # prefill-like
        else:
            counts = np.where(rng.random(E) < 0.5, 0, rng.integers(1, 300, E))   # many empty
        check([int(c) for c in counts], CG, skip_small)


@pytest.mark.parametrize("i", [0, 1, 2, 3])
def test_overlapping_accumulator_epilogue_writes_every_column_once(i):
    """BN = 256 with overlapping accumulators (csrc/gemm_tc.cu, epilogue): tile i accumulates in
    TMEM columns [base, base + 256), base = 128 (i & 1), so consecutive tiles share [128, 256).
    Part 1 reads those shared columns (released at once), part 2 the others; every TMEM column read
    maps to output column (column - base), and each of the 256 output columns is written once."""
    base = 128 * (i & 1)
    p1_tcol, p1_ocol = 128, 128 - base
    p2_tcol, p2_ocol = (0, 0) if base == 0 else (256, 128)
    written = []
    for tcol0, ocol0 in ((p1_tcol, p1_ocol), (p2_tcol, p2_ocol)):
        for c in range(4):                                   # 32-column chunks
            tcol, ocol = tcol0 + 32 * c, ocol0 + 32 * c
            assert base <= tcol < base + 256 and tcol - base == ocol
            written += range(ocol, ocol + 32)
    assert sorted(written) == list(range(256))
    shared = set(range(128, 256))                            # the next tile's accumulator overlaps these
    assert set(range(p1_tcol, p1_tcol + 128)) == shared      # part 1 frees exactly the shared half
    assert base + 256 <= 384                                 # inside the 384 accumulator columns


def epilogue_parts(BN, overlap, i):
    """The epilogue's (TMEM column, output column, width) parts for tile i, as the kernel forms
    them, and the TMEM column the MMAs of tile i start at."""
    base = (i & 1) * 128 if overlap else 0
    d = base
    p1_tcol = 128 if BN == 256 else base
    p1_ocol = 128 - base if BN == 256 else 0
    p2_tcol = 0 if base == 0 else 256
    p2_ocol = 0 if base == 0 else 128
    parts = [(p1_tcol, p1_ocol, 128)]
    if BN == 256:
        parts.append((p2_tcol, p2_ocol, 128))
    return d, parts


@pytest.mark.parametrize("BN,overlap", [(256, True), (256, False), (128, True)])
def test_epilogue_reads_each_output_column_from_its_accumulator_column(BN, overlap):
    """The MMAs of tile i write output column c at TMEM column d + c; the epilogue's parts must
    read exactly those, once each.  With overlapping accumulators (BN = 256) part 1 is the 128
    columns the next tile also writes, so it must be the columns the two tiles share; a part read
    after the release must lie outside the next tile's columns."""
    for i in range(4):
        d, parts = epilogue_parts(BN, overlap, i)
        seen = []
        for tcol, ocol, w in parts:
            for c in range(w):
                assert tcol + c == d + ocol + c
                seen.append(ocol + c)
        assert sorted(seen) == list(range(BN))
        assert d + BN <= (384 if (BN == 256 and overlap) else 256)      # inside the accumulator span
        if BN == 256 and overlap:
            d_next = epilogue_parts(BN, overlap, i + 1)[0]
            nxt = set(range(d_next, d_next + BN))
            assert set(range(parts[0][0], parts[0][0] + 128)) == set(range(d, d + BN)) & nxt
            assert not set(range(parts[1][0], parts[1][0] + 128)) & nxt
        if BN == 128:
            d_next = epilogue_parts(BN, overlap, i + 1)[0]
            assert not set(range(d, d + BN)) & set(range(d_next, d_next + BN))   # two disjoint buffers
