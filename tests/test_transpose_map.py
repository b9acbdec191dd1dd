"""The BF16 transpose of the straight-through backward (csrc/train.cu, ``transpose_bf16_kernel``)
restated on the CPU: 64 x 64 tiles, a load phase (thread t: chunk t % 8 of rows t / 8 and t / 8 + 32)
into a shared tile padded to 66 elements per row, and a store phase (thread t: the 8 rows from
(t % 8) * 8 of columns t / 8 and t / 8 + 32).

Checked for ragged sizes and both store forms: every dst[c][r] = src[r][c] is written exactly once
and nothing outside the R x C block of dst is touched.  The shared-memory bank figures that the
kernel's comment states are recomputed: load-phase writes conflict-free with the padding (4-way
without), store-phase reads at most 2-way (8-way without).
"""
import numpy as np
import pytest

TILE, PAD = 64, 2


def transpose_like_the_kernel(src, R, C, ldd, vec):
    dst = np.full((C, ldd), -1, np.int64)
    writes = np.zeros((C, ldd), np.int64)
    for by in range(-(-R // TILE)):
        for bx in range(-(-C // TILE)):
            r0, c0 = by * TILE, bx * TILE
            tile = np.full((TILE, TILE + PAD), -7, np.int64)
            for t in range(256):
                for rr in range(t >> 3, TILE, 32):
                    cc = (t & 7) * 8
                    r, c = r0 + rr, c0 + cc
                    for j in range(8):
                        tile[rr, cc + j] = src[r, c + j] if (r < R and c + j < C) else 0
            for t in range(256):
                for cc in range(t >> 3, TILE, 32):
                    rr = (t & 7) * 8
                    c, r = c0 + cc, r0 + rr
                    if c >= C:
                        continue
                    v = [tile[rr + j, cc] for j in range(8)]
                    if vec and r + 8 <= R:
                        for j in range(8):
                            dst[c, r + j] = v[j]
                            writes[c, r + j] += 1
                    else:
                        for j in range(8):
                            if r + j < R:
                                dst[c, r + j] = v[j]
                                writes[c, r + j] += 1
    return dst, writes


@pytest.mark.parametrize("R,C", [(1, 1), (7, 130), (64, 64), (65, 63), (200, 9), (128, 192)])
def test_every_element_once_and_nothing_else(R, C):
    rng = np.random.default_rng(R * 1000 + C)
    src = rng.integers(0, 1 << 16, size=(R + TILE, C + TILE))          # reads past R x C must not matter
    for vec in (False, True):
        ldd = R + 8
        dst, writes = transpose_like_the_kernel(src, R, C, ldd, vec)
        assert (dst[:, :R] == src[:R, :C].T).all()
        assert (writes[:, :R] == 1).all() and (writes[:, R:] == 0).all()
        assert (dst[:, R:] == -1).all()


def bank_degree(pad, phase):
    """Worst count of distinct 4-byte words in one bank over the 32 threads of a warp, for any
    one element index j of the 8 each thread moves (2-byte elements, 32 banks)."""
    worst = 0
    for w in range(8):
        for j in range(8):
            banks = {}
            for t in range(32 * w, 32 * w + 32):
                if phase == "store":
                    addr = ((t & 7) * 8 + j) * (TILE + pad) + (t >> 3)
                else:
                    addr = (t >> 3) * (TILE + pad) + (t & 7) * 8 + j
                banks.setdefault((addr // 2) % 32, set()).add(addr // 2)
            worst = max(worst, max(len(v) for v in banks.values()))
    return worst


def test_shared_memory_bank_figures():
    assert bank_degree(PAD, "load") == 1 and bank_degree(0, "load") == 4
    assert bank_degree(PAD, "store") == 2 and bank_degree(0, "store") == 8
