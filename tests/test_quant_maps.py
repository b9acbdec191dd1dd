"""The block quantiser's work map (csrc/quant.cu: ``launch_quantize`` and ``quantize_kernel``),
restated on the CPU: rows per chunk, the chunk-to-CTA distribution (round-robin for the plain
call, contiguous ranges for grouped problems), the chunk's blocks by row passes or by the fp32
row quotient, a grouped chunk's expert and source rows, and the gather of four scales per word.

Checked for K from 64 to 16384 and many batch shapes: every block of every row holding data is
quantised exactly once, into the packed row the grouped layout gives it; padding rows of a grouped
buffer are written as zeros; every scale word's four blocks come from four consecutive threads of
one row.
"""
import numpy as np
import pytest

THREADS, PASS_ROWS = 256, 4


def rows_per_chunk(nb: int) -> tuple[int, bool]:
    passes = nb % THREADS == 0
    if passes:
        return PASS_ROWS, True
    rpc = 1
    while rpc < 128 and rpc * nb < THREADS:
        rpc *= 2
    return rpc, False


def chunk_blocks(nb: int, rpc: int, passes: bool):
    """(thread, row, block) of every block of a chunk, in the kernel's pass order."""
    total = rpc * nb
    out = []
    if passes:
        r, b0 = 0, 0
        for _ in range(0, total, THREADS):
            out += [(t, r, b0 + t) for t in range(THREADS)]
            b0 += THREADS
            if b0 == nb:
                b0, r = 0, r + 1
    else:
        inv = np.float32(1.0) / np.float32(nb)
        for i0 in range(0, total, THREADS):
            for t in range(THREADS):
                i = i0 + t
                if i >= total:
                    continue
                r = int((np.float32(i) + np.float32(0.5)) * inv)
                out.append((t, r, i - r * nb))
    return out


def distribute(nchunks: int, grid: int, grouped: bool):
    if grouped:
        per = -(-nchunks // grid)
        return [list(range(c * per, min(c * per + per, nchunks))) for c in range(grid)]
    return [list(range(c, nchunks, grid)) for c in range(grid)]


def check_scale_words(blocks):
    """Threads 4k .. 4k+3 of a pass hold blocks b .. b+3 (b % 4 == 0) of one row."""
    by_pass = {}
    for n, (t, r, b) in enumerate(blocks):
        by_pass.setdefault(n // THREADS, {})[t] = (r, b)
    for lanes in by_pass.values():
        for t, (r, b) in lanes.items():
            if b % 4 == 0:
                for q in range(1, 4):
                    assert lanes.get(t + q) == (r, b + q), (t, r, b)


@pytest.mark.parametrize("K", [64, 128, 192, 576, 2048, 3072, 4096, 4160, 12288, 16384])
def test_plain_quantiser_covers_every_block_once(K):
    nb = K // 16
    rpc, passes = rows_per_chunk(nb)
    assert 128 % rpc == 0
    blocks = chunk_blocks(nb, rpc, passes)
    assert sorted((r, b) for _, r, b in blocks) == [(r, b) for r in range(rpc) for b in range(nb)]
    check_scale_words(blocks)
    for M in (1, 127, 128, 300, 1000):
        padded = -(-M // 128) * 128
        nchunks = -(-padded // rpc)
        for grid in (1, 7, 148 * 5):
            grid = min(grid, nchunks)
            seen = [0] * nchunks
            for chunks in distribute(nchunks, grid, grouped=False):
                for c in chunks:
                    seen[c] += 1
            assert seen == [1] * nchunks


@pytest.mark.parametrize("K", [64, 512, 2048, 4096])
def test_grouped_quantiser_rows_land_in_the_padded_layout(K):
    """Chunks of rpc packed rows never straddle an expert's 128-row-padded region; a chunk's
    expert is the last with pad[e] <= first row; rows past the expert's count are padding."""
    nb = K // 16
    rpc, _ = rows_per_chunk(nb)
    rng = np.random.default_rng(K)
    for _ in range(40):
        E = int(rng.integers(1, 40))
        counts = [int(c) for c in np.where(rng.random(E) < 0.3, 0, rng.integers(1, 400, E))]
        offs = np.concatenate([[0], np.cumsum(counts)]).tolist()
        pad = np.concatenate([[0], np.cumsum([-(-n // 128) * 128 for n in counts])]).tolist()
        max_rows = offs[-1]
        bound = -(-max_rows // 128) * 128 + 128 * E             # fs_grouped_rows: the launch's rows
        assert pad[-1] <= bound                                 # the layout fits the buffer
        nchunks = -(-bound // rpc)
        written = {}                                           # packed row -> source row or None
        for grid in (3, 148 * 5):
            grid = min(grid, nchunks) if nchunks else 1
            written.clear()
            for chunks in distribute(nchunks, grid, grouped=True):
                for c in chunks:
                    prow0 = c * rpc
                    if prow0 >= pad[-1]:
                        continue
                    e = max(i for i in range(E) if pad[i] <= prow0)
                    local = prow0 - pad[e]
                    assert prow0 + rpc <= pad[e + 1]           # inside the expert's region
                    valid = counts[e] - local
                    for r in range(rpc):
                        assert prow0 + r not in written
                        written[prow0 + r] = offs[e] + local + r if r < valid else None
            for e in range(E):
                for j in range(pad[e], pad[e + 1]):
                    want = offs[e] + (j - pad[e]) if j - pad[e] < counts[e] else None
                    assert written.get(j, "missing") == want, (e, j)


def _mask_tables_like_the_quantiser(words, nb):
    """The per-CTA tables: thread t takes blocks [t per, t per + per), per = ceil(nb / 256); each
    block's 16 mask bits; the side column of its first protected lane from an exclusive scan of the
    per-thread counts; the channel of every side column; per block eight words of lanes to clear."""
    per = -(-nb // THREADS)
    mbits = [(int(words[b >> 1]) >> ((b & 1) * 16)) & 0xFFFF for b in range(nb)]
    col, c = [0] * nb, 0
    for t in range(THREADS):
        for b in range(t * per, min(t * per + per, nb)):
            col[b] = c
            c += bin(mbits[b]).count("1")
    pidx = [0] * 256
    for b in range(nb):
        mb, k = mbits[b], col[b]
        while mb:
            j = (mb & -mb).bit_length() - 1
            mb &= mb - 1
            pidx[k] = b * 16 + j
            k += 1
    kill = []
    for b in range(nb):
        ws = []
        for j in range(8):
            two = (mbits[b] >> (2 * j)) & 3
            ws.append(((two & 1) | ((two & 2) << 15)) * 0xFFFF)
        kill.append(ws)
    return mbits, col, pidx, kill


def test_quantiser_mask_tables():
    """Side columns, channel list and lane kills equal their definitions: the side column of a
    block is the count of protected channels before it, the list is the protected channels in
    ascending order, and the kill words clear exactly the protected bf16 lanes of a block."""
    rng = np.random.default_rng(23)
    for K in (64, 512, 4096, 12288, 16384):
        nb = K // 16
        for p in (0, 1, 16, 64, 256):
            P = np.sort(rng.choice(K, min(p, K), replace=False))
            words = np.zeros(K // 32, np.uint64)
            for j in P:
                words[j // 32] |= np.uint64(1) << np.uint64(j % 32)
            mbits, col, pidx, kill = _mask_tables_like_the_quantiser(words, nb)
            assert col == [int(np.sum(P < 16 * b)) for b in range(nb)]
            assert pidx[:len(P)] == P.tolist()
            for b in rng.integers(0, nb, 20):
                lanes = rng.integers(1, 0xFFFF, 16)              # bf16 bit patterns, none zero
                wordsb = [int(lanes[2 * j]) | (int(lanes[2 * j + 1]) << 16) for j in range(8)]
                cleared = [w & ~k & 0xFFFFFFFF for w, k in zip(wordsb, kill[b])]
                out = [(cleared[j // 2] >> (16 * (j % 2))) & 0xFFFF for j in range(16)]
                prot = {int(j) - 16 * int(b) for j in P if 16 * b <= j < 16 * b + 16}
                assert [out[j] == 0 for j in range(16)] == [j in prot for j in range(16)]
