"""The tensor-core SpliceGEMM's pipeline (csrc/gemm_tc.cu, one CTA) as a protocol model.

Roles and barriers as in the kernel:
* the producer waits on a stage's ``empty`` barrier, then issues the stage's scale atoms (FP4
  k-tiles only, on the stage's ``sfl`` barrier) and its A and B tiles (on ``full``);
* four scale warps, one per TMEM lane quadrant, wait on ``sfl`` (which completes only on the FP4
  uses of a stage, so both sides track its parity per stage), read the atoms, and for each scale
  unit wait on the ring slot's ``sf_empty``, write the slot and arrive on ``sf_full`` (count 4);
* the MMA thread waits on the accumulator's ``acc_empty``, then per k-tile on ``full`` and, per
  scale unit, on ``sf_full``; it commits ``sf_empty`` per unit, ``empty`` per k-tile and
  ``acc_full`` per tile;
* four epilogue warps wait on ``acc_full``, read their quadrant of the accumulator and arrive on
  ``acc_empty`` (count 4): with overlapping accumulators (BN = 256) right after reading the 128
  columns the next tile also writes, without them after the whole tile; with BN = 128 two
  disjoint accumulators take turns, each with its own barrier pair.

Copies land in any order; tensor-core commits complete in issue order.  Every wait uses the
mbarrier rule (a wait for parity P passes once the count of completed phases has the other parity)
and every barrier completes a phase when its expected arrivals (and bytes) are in.  Random
schedules check that nothing is overwritten while it may still be read: a stage's copies wait for
the MMAs and scale warps that read its previous contents, a scale slot for the MMAs of its
previous unit, an accumulator column for the epilogue read of the previous tile that wrote it;
and that every MMA reads its own k-tile and scale unit, every epilogue read its own finished tile,
and nothing deadlocks.  Variants with a known mistake (the scale-atom parity taken from the ring's
phase, the shared columns released before they are read, the wrong half read back) must fail.
"""
import random

import pytest

QUADS = 4


class Bar:
    """An mbarrier: a phase completes when `count` arrivals and every expected copy are in."""

    def __init__(self, count=1):
        self.count, self.done, self.arrived, self.bytes = count, 0, 0, 0

    def ok(self, parity):
        return (self.done & 1) != parity

    def arrive(self, copies=0):
        self.arrived += 1
        self.bytes += copies
        self._maybe_complete()

    def land(self):
        self.bytes -= 1
        self._maybe_complete()

    def _maybe_complete(self):
        if self.arrived == self.count and self.bytes == 0:
            self.done += 1
            self.arrived = 0


ACC_MODES = {
    # name: (accumulator slots, columns a tile writes, read before release, read after release)
    "overlap256": (1, lambda i: [i & 1, (i & 1) + 1], lambda i: [1], lambda i: [2 if i & 1 else 0]),
    "plain256": (1, lambda i: [0, 1], lambda i: [1, 0], lambda i: []),
    "bn128": (2, lambda i: [i & 1], lambda i: [i & 1], lambda i: []),
    # planted mistakes
    "release_first": (1, lambda i: [i & 1, (i & 1) + 1], lambda i: [], lambda i: [1, 2 if i & 1 else 0]),
    "wrong_half": (1, lambda i: [i & 1, (i & 1) + 1], lambda i: [1], lambda i: [0]),
}


def play(S, KT, ST, tiles, sf_bufs, sf_split, acc_mode, seed, sfl_global=False):
    rng = random.Random(seed)
    ktiles = KT + ST
    units = sf_bufs * sf_split
    slots, writes, part1, part2 = ACC_MODES[acc_mode]
    full = [Bar() for _ in range(S)]
    sfl = [Bar() for _ in range(S)]
    empty = [Bar() for _ in range(S)]
    sf_full = [Bar(QUADS) for _ in range(units)]
    sf_empty = [Bar() for _ in range(units)]
    acc_full = [Bar() for _ in range(slots)]
    acc_empty = [Bar(QUADS) for _ in range(slots)]

    stage_ab = [None] * S                     # k-tile whose A/B bytes have landed in a stage
    stage_sf = [None] * S                     # k-tile whose scale atoms have landed in a stage
    ab_issued = [None] * S                    # k-tile whose copies were last issued to a stage
    ab_released = [None] * S                  # k-tile whose MMAs' commit on `empty` completed
    atoms_read = [[None] * S for _ in range(QUADS)]   # k-tile whose atoms each scale warp read
    slot = [[None] * units for _ in range(QUADS)]     # scale unit each quadrant of a slot holds
    slot_released = [None] * units            # unit whose MMAs' commit on `sf_empty` completed
    writer = [dict() for _ in range(QUADS)]   # accumulator column block -> tile that last wrote it
    read = [dict() for _ in range(QUADS)]     # accumulator column block -> tile last read from it
    tiles_done = [-1]                         # last tile whose `acc_full` commit completed
    copies, commits, bad = [], [], []

    def producer():
        stage, phase = 0, 0
        for t in range(tiles):
            for kt in range(ktiles):
                s, ph = stage, phase
                yield lambda: empty[s].ok(ph ^ 1)
                prev = ab_issued[s]
                if prev is not None and ab_released[s] != prev:
                    bad.append(("stage overwritten before its MMAs completed", (t, kt), prev))
                if kt < KT:
                    if prev is not None and prev[1] < KT and any(atoms_read[q][s] != prev for q in range(QUADS)):
                        bad.append(("atoms overwritten before the scale warps read them", (t, kt), prev))
                    sfl[s].arrive(copies=2)                                 # SFA and SFB atoms
                    copies.extend([("sf", s, (t, kt)), ("sf", s, (t, kt))])
                full[s].arrive(copies=2)                                    # A and B tiles
                copies.extend([("ab", s, (t, kt)), ("ab", s, (t, kt))])
                ab_issued[s] = (t, kt)
                stage += 1
                if stage == S:
                    stage, phase = 0, phase ^ 1

    def scale_warp(q):
        stage, phase, unit, bits = 0, 0, 0, 0
        for t in range(tiles):
            for kt in range(ktiles):
                s = stage
                if kt < KT:
                    par = phase if sfl_global else (bits >> s) & 1
                    yield lambda: sfl[s].ok(par)
                    bits ^= 1 << s
                    if stage_sf[s] != (t, kt):
                        bad.append(("scale warp read another k-tile's atoms", (t, kt), stage_sf[s]))
                    atoms_read[q][s] = (t, kt)
                    for h in range(sf_split):
                        u, up = unit % units, ((unit // units) & 1) ^ 1
                        yield lambda: sf_empty[u].ok(up)
                        prev = slot[q][u]
                        if prev is not None and slot_released[u] != prev:
                            bad.append(("scale slot overwritten before its MMAs completed", (t, kt, h), prev))
                        slot[q][u] = (t, kt, h)
                        sf_full[u].arrive()
                        unit += 1
                stage += 1
                if stage == S:
                    stage, phase = 0, phase ^ 1

    def mma_writes(i):
        for q in range(QUADS):
            for c in writes(i):
                w = writer[q].get(c)
                if w is not None and w != i and read[q].get(c) != w:
                    bad.append(("accumulator overwritten before the epilogue read it", i, w))
                writer[q][c] = i

    def mma():
        stage, phase, acc, acc_phase, unit = 0, 0, 0, 0, 0
        for i in range(tiles):
            a, ap = acc, acc_phase
            yield lambda: acc_empty[a].ok(ap ^ 1)
            for kt in range(ktiles):
                s, ph = stage, phase
                yield lambda: full[s].ok(ph)
                if stage_ab[s] != (i, kt):
                    bad.append(("MMA read another k-tile's operands", (i, kt), stage_ab[s]))
                if kt < KT:
                    for h in range(sf_split):
                        u, up = unit % units, (unit // units) & 1
                        yield lambda: sf_full[u].ok(up)
                        if any(slot[q][u] != (i, kt, h) for q in range(QUADS)):
                            bad.append(("MMA read another unit's scales", (i, kt, h), [slot[q][u] for q in range(QUADS)]))
                        mma_writes(i)
                        commits.append(("sf", u, (i, kt, h)))
                        unit += 1
                else:
                    mma_writes(i)
                commits.append(("stage", s, (i, kt)))
                stage += 1
                if stage == S:
                    stage, phase = 0, phase ^ 1
            commits.append(("acc", a, i))
            acc += 1
            if acc == slots:
                acc, acc_phase = 0, acc_phase ^ 1

    def epilogue(q):
        acc, acc_phase = 0, 0
        for i in range(tiles):
            a, ap = acc, acc_phase
            yield lambda: acc_full[a].ok(ap)

            def take(c):
                if writer[q].get(c) != i or tiles_done[0] < i:
                    bad.append(("epilogue read an unfinished or another tile", i, writer[q].get(c), tiles_done[0]))
                read[q][c] = i

            for c in part1(i):
                take(c)
            acc_empty[a].arrive()
            for c in part2(i):
                yield lambda: True                        # the next tile's MMAs may run meanwhile
                take(c)
            acc += 1
            if acc == slots:
                acc, acc_phase = 0, acc_phase ^ 1

    roles = [producer(), mma()] + [scale_warp(q) for q in range(QUADS)] + [epilogue(q) for q in range(QUADS)]
    waits = [None] * len(roles)
    alive = [True] * len(roles)
    for _ in range(1000000):
        for r, role in enumerate(roles):                  # run each released role to its next wait
            if alive[r] and waits[r] is None:
                try:
                    waits[r] = next(role)
                except StopIteration:
                    alive[r] = False
        choices = [r for r in range(len(roles)) if alive[r] and waits[r]()]
        if copies:
            choices.append("copy")
        if commits:
            choices.append("commit")
        if not choices:
            break
        pick = rng.choice(choices)
        if pick == "copy":
            kind, s, ident = copies.pop(rng.randrange(len(copies)))
            if kind == "sf":
                stage_sf[s] = ident
                sfl[s].land()
            else:
                stage_ab[s] = ident
                full[s].land()
        elif pick == "commit":
            kind, k, ident = commits.pop(0)                # tensor-core work completes in order
            if kind == "sf":
                slot_released[k] = ident
                sf_empty[k].arrive()
            elif kind == "stage":
                ab_released[k] = ident
                empty[k].arrive()
            else:
                tiles_done[0] = ident
                acc_full[k].arrive()
        else:
            waits[pick] = None                            # the wait passed; run to the next one
    finished = not any(alive) and not copies and not commits
    return bad, finished


MIXES = [(1, 0), (2, 1), (5, 0), (4, 4), (1, 4), (3, 2)]     # (FP4 k-tiles, BF16 k-tiles)


@pytest.mark.parametrize("acc_mode", ["overlap256", "plain256", "bn128"])
@pytest.mark.parametrize("S", [3, 4, 5])
def test_every_read_sees_its_own_data_and_nothing_deadlocks(acc_mode, S):
    rng = random.Random(S * 7 + len(acc_mode))
    for KT, ST in MIXES:
        for tiles in (1, 2, 5):
            for seed in range(12):
                sf_bufs, sf_split = rng.choice([(2, 1), (1, 1), (2, 2), (2, 4)])
                bad, finished = play(S, KT, ST, tiles, sf_bufs, sf_split, acc_mode, seed)
                assert bad == [] and finished, (acc_mode, S, KT, ST, tiles, sf_bufs, sf_split, seed, bad[:2])


def _fails(**kw):
    for seed in range(200):
        bad, finished = play(seed=seed, **kw)
        if bad or not finished:
            return True
    return False


def test_scale_atom_parity_from_the_ring_phase_goes_wrong():
    """FP4 and BF16 k-tiles mixed so that a stage's uses alternate: the ring's phase no longer
    matches the scale-atom barrier's, and a scale warp reads early or waits forever."""
    assert _fails(S=3, KT=2, ST=2, tiles=3, sf_bufs=2, sf_split=1, acc_mode="overlap256", sfl_global=True)
    assert not _fails(S=3, KT=2, ST=2, tiles=3, sf_bufs=2, sf_split=1, acc_mode="overlap256")


def test_releasing_the_shared_columns_before_reading_them_races():
    assert _fails(S=3, KT=2, ST=1, tiles=4, sf_bufs=2, sf_split=1, acc_mode="release_first")


def test_reading_back_the_wrong_half_is_caught():
    assert _fails(S=3, KT=2, ST=1, tiles=3, sf_bufs=2, sf_split=1, acc_mode="wrong_half")
