"""The decode kernel's in-launch preparation as a protocol model (csrc/gemm_decode_tc.cu, the
kFuse form): R groups of preparing threads fill the stages of a ring of S, group g the k-tiles
g, g + R, ..., each after waiting on the stage's ``empty`` mbarrier with the parity of its use; the
MMA thread consumes the k-tiles in order, each after the stage's ``xfull`` barrier, and its commit
completes the stage's ``empty`` phase.

An mbarrier wait by parity succeeds whenever the number of completed phases has the other parity,
so a waiter two phases behind the barrier passes too soon.  The kernel keeps R <= S, which (its
comment argues) keeps every wait within one phase.  Random schedules are played out with the exact
parity rule: with R <= S the MMA always finds the k-tile it expects in its stage and nothing
deadlocks; with R > S some schedule lets a group overwrite a stage too early.
"""
import random

import pytest


def play(S: int, R: int, nk: int, seed: int):
    """Returns (problems, finished): problems lists the k-tiles the MMA found overwritten."""
    rng = random.Random(seed)
    empty_done = [0] * S            # completed phases of each stage's empty barrier
    xfull_done = [0] * S
    content = [None] * S            # k-tile whose bytes a stage holds
    group_next = list(range(R))     # next k-tile of each group
    mma_next = 0
    pending_commits = []            # stages whose MMAs were issued but not yet completed
    problems = []

    def wait_ok(done, parity):
        return (done & 1) != parity

    for _ in range(100000):
        actions = []
        for g in range(R):
            i = group_next[g]
            if i < nk and wait_ok(empty_done[i % S], ((i // S) & 1) ^ 1):
                actions.append(("group", g))
        if mma_next < nk and wait_ok(xfull_done[mma_next % S], (mma_next // S) & 1):
            actions.append(("mma", None))
        if pending_commits:
            actions.append(("commit", None))
        if not actions:
            break
        kind, g = rng.choice(actions)
        if kind == "group":
            i = group_next[g]
            content[i % S] = i
            xfull_done[i % S] += 1
            group_next[g] = i + R
        elif kind == "mma":
            i = mma_next
            if content[i % S] != i:
                problems.append((i, content[i % S]))
            pending_commits.append(i % S)
            mma_next += 1
        else:
            s = pending_commits.pop(0)   # MMAs complete in issue order
            empty_done[s] += 1
    return problems, mma_next == nk


@pytest.mark.parametrize("R", [1, 2, 3])
def test_at_most_s_groups_keep_every_wait_within_one_phase(R):
    S = 3
    for nk in (1, 2, 3, 4, 7, 16, 20):
        for seed in range(150):
            problems, finished = play(S, R, nk, seed)
            assert problems == [] and finished, (R, nk, seed, problems)


def test_more_groups_than_stages_can_overwrite_a_stage():
    """With R = 2 S a group's parity wait can pass two phases early (the hazard R <= S avoids)."""
    S, R = 3, 6
    assert any(play(S, R, 24, seed)[0] for seed in range(300))
