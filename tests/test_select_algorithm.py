"""The reselection kernel's decision procedure (csrc/stats.cu, ``select_topk_kernel``), restated
step by step on the CPU and checked against the definition of the selection on adversarial keys.

The kernel finds the p-th largest key by a radix select over 8-bit digits from the top, stopping
early once the bin holding the p-th key is taken whole, and then selects every key above the
threshold plus the lowest-index keys equal to it, ranking ties by CTA, warp, round and lane (that
is, by channel index).  A mistake in that logic (a wrong digit scan, an early exit that drops or
adds ties, a tie rank off by one at a CTA boundary) shows up here on key sets chosen to reach every
branch: long runs of equal keys across the threshold, keys equal in every byte but the last, all
keys equal, p = 1 and p = K, K not a multiple of the cluster's 512-channel ranges.  The reference is
the definition itself: the p largest keys, ties to the lower index, in ascending index order.
"""
import numpy as np
import pytest

CLUSTER, THREADS, MAXR = 8, 512, 4


def select_like_the_kernel(keys: np.ndarray, p: int):
    """Threshold search and selection as the kernel does it (all CTAs see the same histograms)."""
    K = len(keys)
    R = -(-K // (CLUSTER * THREADS))
    assert 1 <= R <= MAXR
    T, need = (1 << 64) - 1, 0
    if p > 0:
        prefix, need = 0, p
        for shift in range(56, -1, -8):
            hi_mask = 0 if shift == 56 else ((1 << 64) - 1) ^ ((1 << (shift + 8)) - 1)
            match = (keys & np.uint64(hi_mask)) == np.uint64(prefix)
            digits = ((keys[match] >> np.uint64(shift)) & np.uint64(0xFF)).astype(np.int64)
            tot = np.bincount(digits, minlength=256)
            # the digit holding the need-th largest remaining key: suffix sums from the top
            above, d, binc = 0, None, 0
            for dig in range(255, -1, -1):
                if above < need <= above + tot[dig]:
                    d, binc = dig, int(tot[dig])
                    need -= above
                    break
                above += int(tot[dig])
            assert d is not None
            prefix |= d << shift
            whole_bin = shift > 0 and binc == need
            if whole_bin or shift == 0:
                T = prefix
                if whole_bin:
                    need = p                       # every key equal to T lies in the bin
                break
    # selection in channel order; channel j belongs to CTA j // (512 R), warp, round, lane in order,
    # so the kernel's tie ranks (lower CTAs, warps, rounds, lanes first) are the index order
    sel, ties = [], 0
    for j in range(K):
        k = int(keys[j])
        if k > T:
            sel.append(j)
        elif k == T:
            if ties < need:
                sel.append(j)
            ties += 1
    return np.array(sel, np.int64)


def select_by_definition(keys: np.ndarray, p: int):
    """The p largest keys (exact integer comparison), ties to the lower index, ascending."""
    idx = sorted(range(len(keys)), key=lambda j: (-int(keys[j]), j))[:p]
    return np.array(sorted(idx), np.int64)


def key_sets(rng):
    """Adversarial keys (uint64, as the kernel's order-preserving map would give)."""
    base = np.uint64(0xBFF0000000000000)                  # a positive double's mapped bits
    for K in (64, 96, 1000, 4096, 4100, 12288):
        yield K, rng.integers(0, 1 << 63, K, dtype=np.uint64) | np.uint64(1 << 63)
        yield K, np.full(K, base, np.uint64)                                     # all equal
        yield K, base + rng.integers(0, 4, K, dtype=np.uint64)                   # four values
        yield K, base + (rng.integers(0, 3, K, dtype=np.uint64) << np.uint64(56 - 8))  # differ in one high byte
        k = base + rng.integers(0, 1 << 16, K, dtype=np.uint64)
        k[rng.integers(0, K, K // 4)] = base + np.uint64(777)                    # a long tie run
        yield K, k


@pytest.mark.parametrize("seed", [0, 1])
def test_kernel_selection_logic_matches_the_definition(seed):
    rng = np.random.default_rng(seed)
    for K, keys in key_sets(rng):
        for p in sorted({1, 2, 17, 64, min(256, K), min(K, 256) // 2}):
            if p > K:
                continue
            got = select_like_the_kernel(keys, p)
            want = select_by_definition(keys, p)
            assert len(got) == p and np.array_equal(got, want), (K, p)


def test_kernel_selection_logic_p_equals_k_and_zero():
    keys = np.full(96, np.uint64(0xBFF0000000000000), np.uint64)
    assert np.array_equal(select_like_the_kernel(keys, 96), np.arange(96))
    assert select_like_the_kernel(keys, 0).size == 0


@pytest.mark.parametrize("R", [1, 2, 3, 4])
def test_tie_rank_order_is_channel_order(R):
    """Channel j = rank * 512 R + warp * 32 R + round * 32 + lane (the kernel's mapping): walking
    (rank, warp, round, lane) in order visits 0 .. 4096 R - 1 ascending, so ranking ties by CTA,
    then warp, round and lane ranks them by channel index, and every mask word (32 consecutive
    channels of one round) lies inside one warp."""
    seq = [rank * THREADS * R + warp * 32 * R + r * 32 + lane
           for rank in range(CLUSTER) for warp in range(THREADS // 32) for r in range(R) for lane in range(32)]
    assert seq == list(range(CLUSTER * THREADS * R))
