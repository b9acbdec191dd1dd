"""The tensor-core SpliceGEMM's pipeline (csrc/gemm_tc.cu) as a protocol model, for one CTA and
for a CTA pair (cta_group::2).

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
phase, the shared columns released before they are read, the wrong half read back; in a pair, the
leader's stage barrier expecting only its own bytes, the scale barrier counting one CTA) must fail.
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


def play(S, KT, ST, tiles, sf_bufs, sf_split, acc_mode, seed, cg=1, sfl_global=False, leader_tx=None,
         sf_count=None):
    """One random schedule of a CTA (cg = 1) or a CTA pair (cg = 2); returns (problems, finished).

    In a pair the leader (CTA 0) holds the `full`, `sf_full` and `acc_empty` barriers that count
    both CTAs; the other barriers are per CTA and the leader's commits arrive on both copies.
    `leader_tx` (copies the leader's `full` expects) and `sf_count` plant pair mistakes."""
    rng = random.Random(seed)
    ktiles = KT + ST
    units = sf_bufs * sf_split
    slots, writes, part1, part2 = ACC_MODES[acc_mode]
    ctas = range(cg)
    full = [Bar() for _ in range(S)]                                  # the leader's
    sfl = [[Bar() for _ in range(S)] for _ in ctas]
    empty = [[Bar() for _ in range(S)] for _ in ctas]
    sf_full = [Bar(sf_count or QUADS * cg) for _ in range(units)]     # the leader's
    sf_empty = [[Bar() for _ in range(units)] for _ in ctas]
    acc_full = [[Bar() for _ in range(slots)] for _ in ctas]
    acc_empty = [Bar(QUADS * cg) for _ in range(slots)]               # the leader's

    stage_ab = [[None] * S for _ in ctas]     # k-tile whose A/B bytes have landed in a stage
    stage_sf = [[None] * S for _ in ctas]     # k-tile whose scale atoms have landed in a stage
    ab_issued = [[None] * S for _ in ctas]    # k-tile whose copies were last issued to a stage
    ab_released = [[None] * S for _ in ctas]  # k-tile whose MMAs' commit on `empty` completed
    atoms_read = [[[None] * S for _ in range(QUADS)] for _ in ctas]   # k-tile each scale warp read
    slot = [[[None] * units for _ in range(QUADS)] for _ in ctas]     # unit each quadrant of a slot holds
    slot_released = [[None] * units for _ in ctas]   # unit whose MMAs' commit on `sf_empty` completed
    writer = [[dict() for _ in range(QUADS)] for _ in ctas]   # accumulator column block -> tile that wrote it
    read = [[dict() for _ in range(QUADS)] for _ in ctas]     # accumulator column block -> tile last read
    tiles_done = [-1] * cg                    # last tile whose `acc_full` commit completed
    copies, commits, bad = [], [], []

    def producer(c):
        stage, phase = 0, 0
        for t in range(tiles):
            for kt in range(ktiles):
                s, ph = stage, phase
                yield lambda: empty[c][s].ok(ph ^ 1)
                prev = ab_issued[c][s]
                if prev is not None and ab_released[c][s] != prev:
                    bad.append(("stage overwritten before its MMAs completed", c, (t, kt), prev))
                if kt < KT:
                    if prev is not None and prev[1] < KT and any(atoms_read[c][q][s] != prev for q in range(QUADS)):
                        bad.append(("atoms overwritten before the scale warps read them", c, (t, kt), prev))
                    sfl[c][s].arrive(copies=2)                              # SFA and SFB atoms
                    copies.extend([("sf", c, s, (t, kt))] * 2)
                if c == 0:                                                  # the leader counts both CTAs' bytes
                    full[s].arrive(copies=leader_tx or 2 * cg)
                copies.extend([("ab", c, s, (t, kt))] * 2)                  # A and B tiles
                ab_issued[c][s] = (t, kt)
                stage += 1
                if stage == S:
                    stage, phase = 0, phase ^ 1

    def scale_warp(c, q):
        stage, phase, unit, bits = 0, 0, 0, 0
        for t in range(tiles):
            for kt in range(ktiles):
                s = stage
                if kt < KT:
                    par = phase if sfl_global else (bits >> s) & 1
                    yield lambda: sfl[c][s].ok(par)
                    bits ^= 1 << s
                    if stage_sf[c][s] != (t, kt):
                        bad.append(("scale warp read another k-tile's atoms", c, (t, kt), stage_sf[c][s]))
                    atoms_read[c][q][s] = (t, kt)
                    for h in range(sf_split):
                        u, up = unit % units, ((unit // units) & 1) ^ 1
                        yield lambda: sf_empty[c][u].ok(up)
                        prev = slot[c][q][u]
                        if prev is not None and slot_released[c][u] != prev:
                            bad.append(("scale slot overwritten before its MMAs completed", c, (t, kt, h), prev))
                        slot[c][q][u] = (t, kt, h)
                        sf_full[u].arrive()
                        unit += 1
                stage += 1
                if stage == S:
                    stage, phase = 0, phase ^ 1

    def mma_writes(i):
        for c in ctas:
            for q in range(QUADS):
                for col in writes(i):
                    w = writer[c][q].get(col)
                    if w is not None and w != i and read[c][q].get(col) != w:
                        bad.append(("accumulator overwritten before the epilogue read it", c, i, w))
                    writer[c][q][col] = i

    def mma():
        stage, phase, acc, acc_phase, unit = 0, 0, 0, 0, 0
        for i in range(tiles):
            a, ap = acc, acc_phase
            yield lambda: acc_empty[a].ok(ap ^ 1)
            for kt in range(ktiles):
                s, ph = stage, phase
                yield lambda: full[s].ok(ph)
                for c in ctas:
                    if stage_ab[c][s] != (i, kt):
                        bad.append(("MMA read another k-tile's operands", c, (i, kt), stage_ab[c][s]))
                if kt < KT:
                    for h in range(sf_split):
                        u, up = unit % units, (unit // units) & 1
                        yield lambda: sf_full[u].ok(up)
                        held = [slot[c][q][u] for c in ctas for q in range(QUADS)]
                        if any(x != (i, kt, h) for x in held):
                            bad.append(("MMA read another unit's scales", (i, kt, h), held))
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

    def epilogue(c, q):
        acc, acc_phase = 0, 0
        for i in range(tiles):
            a, ap = acc, acc_phase
            yield lambda: acc_full[c][a].ok(ap)

            def take(col):
                if writer[c][q].get(col) != i or tiles_done[c] < i:
                    bad.append(("epilogue read an unfinished or another tile", c, i, writer[c][q].get(col)))
                read[c][q][col] = i

            for col in part1(i):
                take(col)
            acc_empty[a].arrive()
            for col in part2(i):
                yield lambda: True                        # the next tile's MMAs may run meanwhile
                take(col)
            acc += 1
            if acc == slots:
                acc, acc_phase = 0, acc_phase ^ 1

    roles = [mma()] + [producer(c) for c in ctas]
    roles += [scale_warp(c, q) for c in ctas for q in range(QUADS)] + [epilogue(c, q) for c in ctas for q in range(QUADS)]
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
            kind, c, s, ident = copies.pop(rng.randrange(len(copies)))
            if kind == "sf":
                stage_sf[c][s] = ident
                sfl[c][s].land()
            else:
                stage_ab[c][s] = ident
                full[s].land()
        elif pick == "commit":
            kind, k, ident = commits.pop(0)                # tensor-core work completes in order
            for c in ctas:                                 # the commit arrives on both CTAs' barriers
                if kind == "sf":
                    slot_released[c][k] = ident
                    sf_empty[c][k].arrive()
                elif kind == "stage":
                    ab_released[c][k] = ident
                    empty[c][k].arrive()
                else:
                    tiles_done[c] = ident
                    acc_full[c][k].arrive()
        else:
            waits[pick] = None                            # the wait passed; run to the next one
    finished = not any(alive) and not copies and not commits
    return bad, finished


MIXES = [(1, 0), (2, 1), (5, 0), (4, 4), (1, 4), (3, 2), (0, 1), (0, 5)]   # (FP4, BF16 k-tiles); no FP4: the BF16 GEMM


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


@pytest.mark.parametrize("acc_mode", ["overlap256", "plain256"])
@pytest.mark.parametrize("S", [3, 5])
def test_cta_pairs_read_both_halves_of_their_own_k_tiles(acc_mode, S):
    """cta_group::2: the leader's MMAs read both CTAs' stages and scale slots and write both
    CTAs' accumulators; the peer's copies may land on the leader's barrier before the leader
    has armed it for that phase (its byte count runs below zero until then)."""
    rng = random.Random(S)
    for KT, ST in MIXES:
        for tiles in (1, 2, 4):
            for seed in range(10):
                sf_bufs, sf_split = rng.choice([(2, 1), (1, 1), (2, 2)])
                bad, finished = play(S, KT, ST, tiles, sf_bufs, sf_split, acc_mode, seed, cg=2)
                assert bad == [] and finished, (acc_mode, S, KT, ST, tiles, sf_bufs, sf_split, seed, bad[:2])


def test_a_pair_whose_leader_counts_only_its_own_bytes_races():
    assert _fails(S=3, KT=2, ST=1, tiles=2, sf_bufs=2, sf_split=1, acc_mode="overlap256", cg=2, leader_tx=2)


def test_a_pair_whose_scale_barrier_counts_one_cta_races():
    assert _fails(S=3, KT=3, ST=0, tiles=2, sf_bufs=2, sf_split=1, acc_mode="overlap256", cg=2, sf_count=QUADS)


def play_abort(S, KT, ST, tiles, seed, abort_at, drain):
    """One CTA's pipeline in which a wait gives up at step `abort_at` (the kernel's timeout): the
    flag is raised, every role's pending wait returns false unless its barrier is ready, and each
    role leaves; the producer drains its last min(issued, S) stages by the rule `drain`
    ("always": after its loop, however it ended; "own_failure": only when its own wait gave up;
    "flag_at_finish": only when the flag is up as its loop ends), and the MMA thread waits for all
    it issued.  Returns what is still in flight into the CTA's memory when every role has left."""
    rng = random.Random(seed)
    ktiles = KT + ST
    units = 2
    full, sfl, empty = ([Bar() for _ in range(S)] for _ in range(3))
    sf_full = [Bar(QUADS) for _ in range(units)]
    sf_empty = [Bar() for _ in range(units)]
    acc_full, acc_empty = Bar(), Bar(QUADS)
    copies, commits = [], []
    flag = [False]

    def until(cond):                          # the kernel's wait: ready, or give up once flagged
        return lambda: cond() or flag[0]

    def producer():
        stage, phase, issued, bits, last_fp4 = 0, 0, 0, 0, 0
        ok = True
        for t in range(tiles):
            for kt in range(ktiles):
                s, ph = stage, phase
                ready = lambda: empty[s].ok(ph ^ 1)
                yield until(ready)
                if not ready():
                    ok = False
                    break
                fp4 = kt < KT
                last_fp4 = (last_fp4 & ~(1 << s)) | (int(fp4) << s)
                if fp4:
                    bits ^= 1 << s
                    sfl[s].arrive(copies=2)
                    copies.extend([("sf", s)] * 2)
                full[s].arrive(copies=2)
                copies.extend([("ab", s)] * 2)
                issued += 1
                stage += 1
                if stage == S:
                    stage, phase = 0, phase ^ 1
            if not ok:
                break
        if drain == "always" or (drain == "own_failure" and not ok) or (drain == "flag_at_finish" and flag[0]):
            s, ph = stage, phase
            for _ in range(min(S, issued)):
                s -= 1
                if s < 0:
                    s, ph = S - 1, ph ^ 1
                yield (lambda s=s, ph=ph: full[s].ok(ph))
                if (last_fp4 >> s) & 1:
                    yield (lambda s=s, par=((bits >> s) & 1) ^ 1: sfl[s].ok(par))

    def mma():
        stage, phase, acc_phase, unit = 0, 0, 0, 0
        ok = True
        for _ in range(tiles):
            ap = acc_phase
            ready = lambda: acc_empty.ok(ap ^ 1)
            yield until(ready)
            if not ready():
                break
            for kt in range(ktiles):
                s, ph = stage, phase
                ready = lambda: full[s].ok(ph)
                yield until(ready)
                if not ready():
                    ok = False
                    break
                if kt < KT:
                    u, up = unit % units, (unit // units) & 1
                    ready = lambda: sf_full[u].ok(up)
                    yield until(ready)
                    if not ready():
                        ok = False
                        break
                    commits.append(sf_empty[u])
                    unit += 1
                commits.append(empty[s])
                stage += 1
                if stage == S:
                    stage, phase = 0, phase ^ 1
            if not ok:
                break
            commits.append(acc_full)
            acc_phase ^= 1
        done = Bar()                          # the drain commit: all MMAs issued so far are done
        commits.append(done)
        yield lambda: done.done > 0

    def scale_warp():
        stage, unit, bits = 0, 0, 0
        for _ in range(tiles):
            for kt in range(ktiles):
                s = stage
                if kt < KT:
                    par = (bits >> s) & 1
                    ready = lambda: sfl[s].ok(par)
                    yield until(ready)
                    if not ready():
                        return
                    bits ^= 1 << s
                    u, up = unit % units, ((unit // units) & 1) ^ 1
                    ready = lambda: sf_empty[u].ok(up)
                    yield until(ready)
                    if not ready():
                        return
                    sf_full[u].arrive()
                    unit += 1
                stage = (stage + 1) % S

    def epilogue():
        acc_phase = 0
        for _ in range(tiles):
            ap = acc_phase
            ready = lambda: acc_full.ok(ap)
            yield until(ready)
            if not ready():
                return
            acc_empty.arrive()
            acc_phase ^= 1

    roles = [producer(), mma()] + [scale_warp() for _ in range(QUADS)] + [epilogue() for _ in range(QUADS)]
    waits = [None] * len(roles)
    alive = [True] * len(roles)
    for step in range(1, 1000000):
        for r, role in enumerate(roles):
            if alive[r] and waits[r] is None:
                try:
                    waits[r] = next(role)
                except StopIteration:
                    alive[r] = False
        if not any(alive):
            break
        if step == abort_at:
            flag[0] = True
        choices = [r for r in range(len(roles)) if alive[r] and waits[r]()]
        if copies:
            choices.append("copy")
        if commits:
            choices.append("commit")
        assert choices, "deadlock"
        pick = rng.choice(choices)
        if pick == "copy":
            kind, s = copies.pop(rng.randrange(len(copies)))
            (sfl if kind == "sf" else full)[s].land()
        elif pick == "commit":
            commits.pop(0).arrive()
        else:
            waits[pick] = None
    return len(copies), len(commits)


def _abort_cases(n):
    rng = random.Random(2024)
    for seed in range(n):
        KT, ST = rng.choice([(2, 1), (4, 0), (1, 3), (3, 3), (5, 2)])
        yield rng.choice([3, 4, 5]), KT, ST, rng.choice([1, 2, 3]), seed, rng.randrange(1, 90)


def test_after_a_timeout_nothing_is_in_flight_when_the_cta_exits():
    """Both kernels' producers drain after their loop however it ended, so a CTA that gave up
    exits with no copy landing in its shared memory and no MMA running, wherever the timeout
    fell (also after the producer had issued everything, or before anything was issued)."""
    for S, KT, ST, tiles, seed, abort_at in _abort_cases(1500):
        assert play_abort(S, KT, ST, tiles, seed, abort_at, "always") == (0, 0), (S, KT, ST, tiles, seed, abort_at)


@pytest.mark.parametrize("drain", ["own_failure", "flag_at_finish"])
def test_draining_only_on_the_producers_own_failure_can_leave_copies_in_flight(drain):
    """The narrower rules miss a timeout that falls after the producer's loop has ended."""
    assert any(play_abort(*case, drain)[0] for case in _abort_cases(1500))
