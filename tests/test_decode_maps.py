"""Index arithmetic of the decode kernel (csrc/gemm_decode_tc.cu and its launcher), restated on
the CPU: the K split over a cluster, the cluster reduction's output shares, the fused
preparation's k-tile schedule and the bytes it writes into a stage's scale atoms.  The GPU parity
tests check the results; these check that every piece of work has exactly one owner for every
shape the launcher can choose, including shapes the GPU tests do not reach.
"""
import pytest

from oracle import nvfp4

KD_ROWS, KD_TOK, MAX_SPLIT, STAGES = 128, 16, 8, 3


def k_split(KT: int, tiles: int, slots: int = 3 * 148):
    """The launcher's split: as many CTAs per tile as fill the resident slots, at most 8, every
    CTA with at least one FP4 k-tile."""
    S = max(1, slots // tiles)
    S = min(S, min(MAX_SPLIT, KT))
    kt_per = -(-KT // S)
    S = -(-KT // kt_per)
    return S, kt_per


@pytest.mark.parametrize("KT", list(range(1, 65)) + [96, 128, 192, 256])
def test_k_split_gives_every_rank_fp4_k_tiles_and_covers_k(KT):
    for tiles in (1, 2, 8, 32, 48, 96, 192, 444, 2048):
        S, kt_per = k_split(KT, tiles)
        owned = []
        for rank in range(S):
            kt0 = rank * kt_per
            kt1 = min(kt0 + kt_per, KT)
            assert kt1 > kt0, (KT, tiles, rank)                    # nf >= 1
            owned += range(kt0, kt1)
        assert owned == list(range(KT))


@pytest.mark.parametrize("S", range(1, MAX_SPLIT + 1))
def test_cluster_reduction_shares_write_every_output_once(S):
    """Outputs v = token * 128 + row of a tile, four per thread step; CTA rank takes
    [rank * share, min((rank + 1) * share, 2048)) with share rounded up to a multiple of 4, and
    thread e of the 128 epilogue threads the groups of four from rank * share + 4 e on."""
    k_out = KD_ROWS * KD_TOK
    share = (-(-k_out // S) + 3) & ~3
    seen = [0] * k_out
    for rank in range(S):
        v0, v1 = rank * share, min(rank * share + share, k_out)
        for e in range(128):
            for v in range(v0 + 4 * e, v1, 4 * 128):
                for q in range(4):
                    seen[v + q] += 1
    assert seen == [1] * k_out


@pytest.mark.parametrize("M", range(1, KD_TOK + 1))
def test_fused_preparation_schedule(M):
    """Groups of 8 M threads, R = min(128 / (8 M), stages) of them: group g prepares the FP4 k-tiles
    g, g + R, ... and then the side k-tiles i >= nf with i = g (mod R); every k-tile of the CTA has
    exactly one group, and a group's consecutive k-tiles are at most R <= stages apart (so its
    stage waits stay within one phase)."""
    G = 8 * M
    R = min(128 // G, STAGES)
    assert 1 <= R <= STAGES
    for nf in range(1, 20):
        for st in range(0, 5):
            nk = nf + st
            owner = {}
            for g in range(R):
                mine = list(range(g, nf, R))
                i = nf + ((g - nf % R) % R + R) % R
                while i < nk:
                    mine.append(i)
                    i += R
                for a, b in zip(mine, mine[1:]):
                    assert 0 < b - a <= R
                for i in mine:
                    assert i not in owner
                    owner[i] = g
            assert sorted(owner) == list(range(nk)), (M, nf, st)


def test_fused_preparation_scale_bytes_follow_the_tiled_layout():
    """Thread (r, c) of a group encodes blocks 2c and 2c + 1 of token row r in a k-tile and writes
    their two scale bytes at 512 (c >> 1) + 16 r + (2c & 3) of the stage's four atoms: the bytes the
    tiled scale layout gives those (row, block) pairs, relative to the k-tile's first atom."""
    K = 4096
    for kt in (0, 1, 7, 15):
        base = kt * 4 * 512                                     # the k-tile's atoms (row group 0)
        for r in range(KD_TOK):
            for c in range(8):
                off = 512 * (c >> 1) + r * 16 + ((2 * c) & 3)
                for h in range(2):
                    b = kt * 16 + 2 * c + h
                    assert int(nvfp4.sf_tiled_offset(r, b, K)) - base == off + h


def test_fused_preparation_x_swizzle_is_the_128_byte_pattern():
    """Chunk c (16 bytes: channels 32c .. 32c+31 as E2M1 codes) of token row r goes to byte
    128 r + 16 (c ^ (r mod 8)) of the X box: the 128-byte swizzle, a permutation of each row's
    eight chunks."""
    for r in range(KD_TOK):
        offs = sorted(128 * r + 16 * (c ^ (r & 7)) for c in range(8))
        assert offs == [128 * r + 16 * j for j in range(8)]


def _protected_list_like_the_decode_prep(words, KT):
    """The fused preparation's channel list: 128 threads take contiguous ranges of the K/32 mask
    words (ceil(nw / 128) each), count their set bits, scan the counts in thread order and write
    their channels in ascending order from that position (positions past 256 dropped)."""
    nw = KT * 8
    per = -(-nw // 128)
    counts, ranges = [], []
    for t in range(128):
        w0 = min(t * per, nw)
        w1 = min(w0 + per, nw)
        ranges.append((w0, w1))
        counts.append(sum(bin(int(words[w])).count("1") for w in range(w0, w1)))
    pidx = [0] * 256
    pos = 0
    for t in range(128):
        w0, w1 = ranges[t]
        for w in range(w0, w1):
            mw = int(words[w])
            while mw:
                b = (mw & -mw).bit_length() - 1
                mw &= mw - 1
                if pos < 256:
                    pidx[pos] = w * 32 + b
                pos += 1
    assert pos == sum(counts)
    return pidx, pos


def test_decode_prep_protected_channel_list():
    """The list equals the protected channels in ascending order (the side columns' order) for
    random sets of up to 256 channels, K from 256 to 16384 (per-thread ranges of 1 to 4 words)."""
    import numpy as np
    rng = np.random.default_rng(21)
    for K in (256, 512, 4096, 12288, 16384):
        for p in (0, 1, 17, 64, 256):
            P = np.sort(rng.choice(K, p, replace=False))
            words = np.zeros(K // 32, np.uint64)
            for j in P:
                words[j // 32] |= np.uint64(1) << np.uint64(j % 32)
            pidx, n = _protected_list_like_the_decode_prep(words, K // 256)
            assert n == p and pidx[:p] == P.tolist()
