"""The reselection kernel's histogram exchange (csrc/stats.cu, ``select_topk_kernel``) as a
protocol model: each of the 8 CTAs of a cluster, in every radix pass i, clears its histogram
buffer i % 2, accumulates into it, arrives at and waits on the cluster barrier of pass i, then reads
buffer i % 2 of every CTA through distributed shared memory.  The kernel's claim is that one barrier
per pass suffices with two buffers: no CTA rewrites a buffer while another may still read it.

Random schedules (any interleaving the barrier allows) are played out, and every remote read
must see the owner's histogram of the same pass.  The same model with a single buffer is shown
to race, so the check has teeth.
"""
import random

import pytest

CTAS = 8


def play(passes: int, buffers: int, seed: int) -> list:
    """Runs one random schedule; returns the reads that saw another pass's histogram."""
    rng = random.Random(seed)
    # per CTA, the program: (op, pass) with ops clear, acc, barrier, read(c) for every c
    progs = []
    for _ in range(CTAS):
        prog = []
        for i in range(passes):
            prog += [("clear", i), ("acc", i), ("barrier", i)] + [("read", i, c) for c in range(CTAS)]
        prog.append(("barrier", passes))              # the kernel's later barriers (counts, exit)
        progs.append(prog)
    pc = [0] * CTAS
    arrived = {}                                      # barrier id -> set of CTAs that arrived
    content = {}                                      # (cta, buffer) -> (pass, complete)
    bad = []
    while any(pc[c] < len(progs[c]) for c in range(CTAS)):
        ready = []
        for c in range(CTAS):
            if pc[c] >= len(progs[c]):
                continue
            op = progs[c][pc[c]]
            if op[0] == "barrier":
                arrived.setdefault(op[1], set()).add(c)
                if len(arrived[op[1]]) < CTAS:
                    continue                          # waits until every CTA has arrived
            ready.append(c)
        assert ready, "deadlock"
        c = rng.choice(ready)
        op = progs[c][pc[c]]
        pc[c] += 1
        if op[0] == "clear":
            content[(c, op[1] % buffers)] = (op[1], False)
        elif op[0] == "acc":
            content[(c, op[1] % buffers)] = (op[1], True)
        elif op[0] == "read":
            _, i, owner = op
            if content.get((owner, i % buffers)) != (i, True):
                bad.append((c, owner, i, content.get((owner, i % buffers))))
    return bad


@pytest.mark.parametrize("passes", [1, 2, 3, 8])
def test_double_buffered_histograms_need_one_barrier_per_pass(passes):
    for seed in range(400):
        assert play(passes, buffers=2, seed=seed) == []


def test_a_single_buffer_would_race():
    assert any(play(3, buffers=1, seed=s) for s in range(400))
