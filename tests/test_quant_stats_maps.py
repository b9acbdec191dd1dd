"""The fused statistics-and-quantise kernel's work map (csrc/quant_stats.cu: ``quantize_stats_kernel``
and ``launch_quantize_rows``), restated on the CPU and checked against what it must cover.

* Rows: CTA (x, y) holds the 256-channel slab x; its warp w takes the row pairs starting at
  2 (8 y + w), stepping by 16 gy.  Every row of the 128-padded batch must be taken once per slab,
  for every grid height the launcher can pick.
* The per-warp ring of 4 row pairs filled by cp.async: one commit group per iteration (empty past
  the batch), ``wait_group 3`` before reading.  The slot a warp reads must hold that iteration's
  rows with its group complete, and a slot must not be refilled before its rows were read.
* ``r0 mod row_stride`` kept incrementally; the rows the statistics take (row % row_stride == 0,
  before masking, FourSight §5.2) once each, and the row count the kernel adds to n.
* Each lane's 8 channels: its protected lanes, the side column of its first protected channel (a
  warp-summed popcount of the slab's earlier mask words plus its own), the kill words, and the
  zeroed padding side columns; and the scale word of blocks 4k .. 4k+3 gathered from lanes 8k,
  8k+2, 8k+4, 8k+6 (a 16-element block is two adjacent lanes).
"""
import numpy as np
import pytest

WARPS, SLAB, DEPTH = 8, 256, 4


def ceil_div(a, b):
    return -(-a // b)


def launch_grid(K, Mp, slots, sms):
    chunks = ceil_div(K, SLAB)
    gy = max(1, slots * sms // chunks)
    gy = min(gy, max(1, ceil_div(Mp, 2 * WARPS * 16)))
    return chunks, min(gy, 65535)


def warp_rows(y, w, gy, Mp):
    step = gy * WARPS * 2
    return list(range((y * WARPS + w) * 2, Mp, step))


@pytest.mark.parametrize("K", [64, 4096, 12288, 16384])
def test_every_row_pair_is_taken_once_per_slab(K):
    for M in (1, 2, 127, 128, 129, 1000, 8192, 20000):
        Mp = ceil_div(M, 128) * 128
        for slots, sms in ((1, 1), (2, 148), (3, 148), (2, 7)):
            _, gy = launch_grid(K, Mp, slots, sms)
            seen = np.zeros(Mp, np.int64)
            for y in range(gy):
                for w in range(WARPS):
                    for r0 in warp_rows(y, w, gy, Mp):
                        seen[r0] += 1
                        seen[r0 + 1] += 1
            assert (seen == 1).all(), (K, M, slots, sms, gy)


def test_the_cp_async_ring_reads_each_pair_once_it_has_landed():
    """Groups complete in commit order; wait_group(3) leaves only the 3 newest pending."""
    for M, gy in ((1, 1), (128, 1), (1000, 3), (8192, 5), (300, 40)):
        Mp = ceil_div(M, 128) * 128
        step = gy * WARPS * 2
        for first in (0, 2, 14, 2 * (gy * WARPS - 1)):
            if first >= Mp:
                continue
            slot_rows = [None] * DEPTH            # row pair a slot was last filled with
            slot_group = [None] * DEPTH
            slot_read = [True] * DEPTH            # its rows were read since the fill
            groups_done, groups = 0, 0

            def issue(r0, s):
                nonlocal groups
                if r0 < M:                        # rows past the batch are not copied
                    assert slot_read[s], "a slot refilled before its rows were read"
                    slot_rows[s], slot_group[s], slot_read[s] = r0, groups, False
                groups += 1                       # the commit group is made either way

            for d in range(DEPTH - 1):
                issue(first + d * step, d)
            slot = 0
            for r0 in range(first, Mp, step):
                issue(r0 + (DEPTH - 1) * step, (slot + DEPTH - 1) % DEPTH)
                groups_done = max(groups_done, groups - (DEPTH - 1))     # cp.async.wait_group 3
                if r0 < M:
                    assert slot_rows[slot] == r0 and slot_group[slot] < groups_done
                    slot_read[slot] = True
                slot = (slot + 1) % DEPTH


def test_incremental_row_modulus_and_the_rows_the_statistics_take():
    rng = np.random.default_rng(5)
    for _ in range(300):
        M = int(rng.integers(1, 5000))
        Mp = ceil_div(M, 128) * 128
        stride = int(rng.choice([1, 2, 3, 7, 16, 100, 129, 4096, 10000]))
        gy = int(rng.integers(1, 12))
        step = gy * WARPS * 2
        taken = []
        for y in range(gy):
            for w in range(WARPS):
                first = (y * WARPS + w) * 2
                mod0, dmod = first % stride, step % stride
                for r0 in range(first, Mp, step):
                    mod1 = 0 if mod0 + 1 == stride else mod0 + 1
                    assert (mod0, mod1) == (r0 % stride, (r0 + 1) % stride)
                    if r0 < M and mod0 == 0:
                        taken.append(r0)
                    if r0 + 1 < M and mod1 == 0:
                        taken.append(r0 + 1)
                    mod0 += dmod
                    if mod0 >= stride:
                        mod0 -= stride
        assert sorted(taken) == list(range(0, M, stride))
        assert len(taken) == ceil_div(M, stride)             # what the kernel adds to n


def lane_view(words, K, x, lane):
    """(active, protected bits of the lane's 8 channels, protected channels below its first),
    computed the kernel's way."""
    c0 = x * SLAB + lane * 8
    active = c0 < K
    slab_w = (x * SLAB) >> 5
    below = 0
    for w0 in range(0, slab_w, 32):                      # the warp sums 32 words per step
        below += sum(bin(int(words[w])).count("1") for w in range(w0, min(w0 + 32, slab_w)))
    pbits = 0
    if active:
        wi = c0 >> 5
        below += sum(bin(int(words[w])).count("1") for w in range(slab_w, wi))
        mw = int(words[wi])
        below += bin(mw & ((1 << (c0 & 31)) - 1)).count("1")
        pbits = (mw >> (c0 & 31)) & 0xFF
    return active, pbits, below


@pytest.mark.parametrize("K", [64, 320, 4096, 12288, 16384])
def test_lane_protected_bits_side_columns_and_kills(K):
    rng = np.random.default_rng(K)
    for p in (0, 1, 7, 64, 256):
        P = np.sort(rng.choice(K, min(p, K), replace=False))
        words = np.zeros(K // 32, np.uint64)
        for j in P:
            words[j // 32] |= np.uint64(1) << np.uint64(j % 32)
        pset = set(P.tolist())
        side = {}                                        # side column -> channel
        for x in range(ceil_div(K, SLAB)):
            for lane in range(32):
                active, pbits, col0 = lane_view(words, K, x, lane)
                c0 = x * SLAB + lane * 8
                assert active == (c0 < K)
                if not active:
                    continue
                assert col0 == int(np.sum(P < c0))
                assert [(pbits >> j) & 1 for j in range(8)] == [int(c0 + j in pset) for j in range(8)]
                kill = []
                for j in range(4):
                    two = (pbits >> (2 * j)) & 3
                    kill.append(((two & 1) | ((two & 2) << 15)) * 0xFFFF)
                for vals in ([0xFFFF] * 8, rng.integers(1, 0x10000, 8).tolist()):   # nonzero bf16 patterns
                    words4 = [vals[2 * j] | (vals[2 * j + 1] << 16) for j in range(4)]
                    kept = [(words4[j // 2] & ~kill[j // 2] & 0xFFFFFFFF) >> (16 * (j % 2)) & 0xFFFF for j in range(8)]
                    assert [v == 0 for v in kept] == [c0 + j in pset for j in range(8)]
                    assert all(v in (0, w) for v, w in zip(kept, vals))  # a kept lane is untouched
                col = col0
                pb = pbits
                while pb:
                    j = (pb & -pb).bit_length() - 1
                    pb &= pb - 1
                    assert col not in side
                    side[col] = c0 + j
                    col += 1
        assert side == dict(enumerate(P.tolist()))       # X_S column k holds the k-th protected channel
        pp = (len(P) + 15) // 16 * 16
        assert 0 <= pp - len(P) <= 32 - 1                # slab 0's lanes zero the padding columns


@pytest.mark.parametrize("K", [64, 192, 4096, 16384])
def test_scale_words_gather_four_consecutive_blocks(K):
    """Lane 8k writes the word of blocks 4k' .. 4k'+3 of its slab row from itself and lanes
    8k+2, 8k+4, 8k+6; active lanes come in whole groups of 8 (K % 64 == 0)."""
    kb4 = ceil_div(K // 16, 4)
    for x in range(ceil_div(K, SLAB)):
        blk = [(x * SLAB + lane * 8) >> 4 for lane in range(32)]
        act = [x * SLAB + lane * 8 < K for lane in range(32)]
        for k in range(4):
            assert len(set(act[8 * k:8 * k + 8])) == 1
            if not act[8 * k]:
                continue
            b0 = blk[8 * k]
            assert b0 % 4 == 0 and [blk[8 * k + 2 * i] for i in range(4)] == [b0 + i for i in range(4)]
            assert blk[8 * k + 1] == b0                  # the partner lane of a block
            for r in (0, 31, 32, 127, 128, 1000):
                off = ((r >> 7) * kb4 + (b0 >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4
                assert off % 4 == 0                      # a whole aligned 32-bit word per (row, 4 blocks)
