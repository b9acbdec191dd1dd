"""The sequence filter's run reduction (csrc/filter.cu: ``push``, ``combine`` and the kernel's
ordered reduction), restated on the CPU and checked against a direct count of tail tokens and of
the longest run of consecutive tail tokens (FourSight §4.1, Eq. 3).

Each of 256 threads summarises a contiguous chunk of 4 * ceil(L / 1024) tokens; lane summaries
combine in a shuffle-down tree (lane l takes lane l + o when l is a multiple of 2 o), then the
eight warp results combine in order.  Random tail masks of every kind are used: runs that cross
thread and warp boundaries, all tail, no tail, a single tail token at either end, lengths that do
not fill the last chunk.
"""
import numpy as np
import pytest

THREADS = 256


def empty():
    return [0, 0, 0, 0, 0]                     # len, cnt, pre, suf, best


def push(s, tail):
    if tail:
        s[1] += 1
        if s[2] == s[0]:
            s[2] += 1
        s[3] += 1
        s[4] = max(s[4], s[3])
    else:
        s[3] = 0
    s[0] += 1


def combine(a, b):
    return [a[0] + b[0], a[1] + b[1],
            a[0] + b[2] if a[2] == a[0] else a[2],
            b[0] + a[3] if b[3] == b[0] else b[3],
            max(a[4], b[4], a[3] + b[2])]


def reduce_like_the_kernel(mask):
    L = len(mask)
    per4 = -(-L // (4 * THREADS))
    acc = []
    for tid in range(THREADS):
        s = empty()
        t0 = tid * per4 * 4
        for t in range(t0, min(t0 + 4 * per4, L)):
            push(s, bool(mask[t]))
        acc.append(s)
    warps = []
    for w in range(THREADS // 32):
        lanes = [list(x) for x in acc[32 * w:32 * w + 32]]
        o = 1
        while o < 32:
            before = [list(x) for x in lanes]                 # every lane shuffles its current value
            for lane in range(32):
                if lane + o < 32 and lane % (2 * o) == 0:
                    lanes[lane] = combine(before[lane], before[lane + o])
            o *= 2
        warps.append(lanes[0])
    tot = warps[0]
    for w in warps[1:]:
        tot = combine(tot, w)
    return tot


def direct(mask):
    cnt = int(np.sum(mask))
    best = run = 0
    for m in mask:
        run = run + 1 if m else 0
        best = max(best, run)
    return cnt, best


@pytest.mark.parametrize("seed", range(4))
def test_run_reduction_matches_a_direct_count(seed):
    rng = np.random.default_rng(seed)
    for L in [0, 1, 3, 4, 5, 1023, 1024, 1025, 4096, 4100, 8192]:
        masks = [np.zeros(L, bool), np.ones(L, bool), rng.random(L) < 0.02, rng.random(L) < 0.5]
        if L:
            one = np.zeros(L, bool); one[0] = True; masks.append(one)
            last = np.zeros(L, bool); last[-1] = True; masks.append(last)
            runs = np.zeros(L, bool)                          # runs across chunk and warp boundaries
            for start in rng.integers(0, L, 6):
                runs[start:start + int(rng.integers(1, 700))] = True
            masks.append(runs)
        for m in masks:
            tot = reduce_like_the_kernel(m)
            assert tot[0] == L
            assert (tot[1], tot[4]) == direct(m), (L, seed)
