"""Host model of the synchronisation inside one CTA of the GEMV kernel
(q4_gemv.cuh): a producer filling an S-stage ring (bulk copies that land in
any order), sixteen consumer warps (column 0 / 1 x block index 0..7) that
take every stage and, at each row block segment's end, hand their sums to
the epilogue through reduction buffers, and two epilogue warps.  Two slot
layouts: one slot per consumer warp (M <= 3), or one per block index with
the column-1 warp adding to what the column-0 warp stored ("pair slots",
M >= 4).  Random interleavings must always finish; every parity wait must
start while its barrier is at the awaited phase or one past it; a stage is
read only while it holds its unit; a slot is written only after the epilogue
has read its previous contents; a column-1 warp adds only to its partner's
sums of the same segment; and the epilogue reads exactly the sixteen
contributions of its segment.  Mistakes planted in the model (a dropped
wait, a wrong barrier count) must make it fail."""
import random

import pytest

WARPS = 16


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.arrived, self.phase = name, count, 0, 0

    def arrive(self):
        self.arrived += 1
        assert self.arrived <= self.count, self.name
        if self.arrived == self.count:
            self.arrived = 0
            self.phase += 1


def simulate(segments, S, bufs, pair, seed, mistake=None):
    rnd = random.Random(seed)
    units = [(seg, k) for seg, n in enumerate(segments) for k in range(n)]
    full = [Bar(f"full{s}", 1) for s in range(S)]
    empty = [Bar(f"empty{s}", WARPS) for s in range(S)]
    red_full_count = 8 if pair and mistake != "red_full_counts_every_warp" else 16
    red_full = [Bar(f"red_full{b}", red_full_count) for b in range(bufs)]
    red_empty = [Bar(f"red_empty{b}", 2) for b in range(bufs)]
    red_pair = [[Bar(f"pair{b}.{k}", 1) for k in range(8)] for b in range(bufs)]
    n_slots = 8 if pair else 16
    slots = [[None] * n_slots for _ in range(bufs)]   # (segment, set of contributions)
    ring = [None] * S
    reads = {}                                           # segment -> epilogue warps done
    pending = []

    def wait(bar, k):
        assert k <= bar.phase <= k + 1, (bar.name, k, bar.phase)
        while bar.phase <= k:
            yield

    def producer():
        for i, u in enumerate(units):
            slot = i % S
            if i >= S:
                yield from wait(empty[slot], i // S - 1)
            ring[slot] = u
            pending.append(slot)
            yield

    def consumer(w):
        col, blk = w >> 3, w & 7
        i = 0
        for seg, n in enumerate(segments):
            for k in range(n):
                slot = i % S
                yield from wait(full[slot], i // S)
                assert ring[slot] == (seg, k), "stage overwritten before every warp read it"
                yield
                empty[slot].arrive()
                i += 1
            b = seg % bufs
            if seg >= bufs and mistake != "no_red_empty_wait":
                yield from wait(red_empty[b], (seg - bufs) // bufs)
            s = blk if pair else w
            if pair and col == 1:
                if mistake != "no_pair_wait":
                    yield from wait(red_pair[b][blk], seg // bufs)
                cur = slots[b][s]
                assert cur is not None and cur[0] == seg and cur[1] == {(0, blk)}, \
                    "column 1 added to something other than its partner's sums"
                yield
                slots[b][s] = (seg, cur[1] | {(1, blk)})
                red_full[b].arrive()
            else:
                prev = slots[b][s]
                assert prev is None or reads.get(prev[0], 0) == 2, \
                    "slot rewritten before the epilogue read it"
                yield
                slots[b][s] = (seg, {(col, blk)})
                if pair:
                    red_pair[b][blk].arrive()
                else:
                    red_full[b].arrive()
            yield

    def epilogue(e):
        for seg in range(len(segments)):
            b = seg % bufs
            yield from wait(red_full[b], seg // bufs)
            got = set()
            for sl in slots[b]:
                assert sl is not None and sl[0] == seg, "epilogue read another segment's slot"
                got |= sl[1]
            assert got == {(c, k) for c in range(2) for k in range(8)}
            yield
            reads[seg] = reads.get(seg, 0) + 1
            red_empty[b].arrive()
            yield

    actors = {"producer": producer()}
    for w in range(WARPS):
        actors[("c", w)] = consumer(w)
    for e in range(2):
        actors[("e", e)] = epilogue(e)
    speed = {a: rnd.choice([0.05, 1.0, 1.0, 4.0]) for a in actors}
    speed["copy"] = rnd.choice([0.1, 1.0, 4.0])
    steps = 0
    while actors or pending:
        steps += 1
        assert steps < 300000, "no progress"
        choices = list(actors) + ["copy"] * bool(pending)
        assert choices, "deadlock"
        c = rnd.choices(choices, weights=[speed[x] for x in choices])[0]
        if c == "copy":
            full[pending.pop(rnd.randrange(len(pending)))].arrive()
            continue
        try:
            next(actors[c])
        except StopIteration:
            del actors[c]
    assert all(reads.get(seg) == 2 for seg in range(len(segments)))


SEGMENTS = [[1], [3], [1, 1, 1, 1], [2, 5, 1, 3], [10, 1, 10], [1, 4, 1, 4, 1, 4, 1]]


@pytest.mark.parametrize("segments", SEGMENTS)
@pytest.mark.parametrize("S,bufs,pair", [(5, 2, False), (5, 1, False), (2, 1, False),
                                         (5, 1, True), (2, 1, True), (4, 2, True)])
def test_gemv_cta_protocol(segments, S, bufs, pair):
    for seed in range(12):
        simulate(segments, S, bufs, pair, seed)


@pytest.mark.parametrize("mistake", ["no_pair_wait", "no_red_empty_wait",
                                     "red_full_counts_every_warp"])
def test_planted_mistakes_fail(mistake):
    for seed in range(40):
        try:
            simulate([2, 1, 3, 1, 2], 3, 1, True, seed, mistake)
        except AssertionError:
            return
    raise AssertionError(f"the model did not catch {mistake}")
