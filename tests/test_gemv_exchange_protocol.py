"""Host model of the GEMV's protocol between CTAs (q4_gemv.cuh), launch after
launch over the same workspace and descriptor: the stream-K partition of
each job's units (rotated by the units of the jobs before it), the finisher
of a shared row block (the CTA whose range ends in it: slot 0), the other
contributors' partial sums published as tagged entries, the finisher
reading them once they carry the launch's tag, adding them in slot order,
clearing them and counting the row block for its job; a job's activations
are read only once the job it waits for has counted all of its row blocks;
the last CTA to leave sets the counters back to zero.

Random schedules over several launches -- the second a replay with the same
tag, as a captured graph would be -- must finish with every row block the
sum of exactly its own units of this launch, no dependent job started before
its input was complete, and the workspace and counters left zero.  Mistakes
planted in the model (no clearing, no counter reset, untagged entries, no
wait for the tag, a row block counted before it is written) must make it
fail."""
import random

import pytest


def _unit_begin(c, U, G):
    return c * U // G


def _unit_owner(u, U, G):
    return ((u + 1) * G - 1) // U


def _plan(shapes, G):
    """Job descriptors as the host prepares them: (rbs, upr, wait_for) each."""
    jobs, before, part_off = [], 0, 0
    for rbs, upr, wait_for in shapes:
        U = rbs * upr
        g = min(G, U)
        slots = 0
        for rb in range(rbs):
            first, last = _unit_owner(rb * upr, U, g), _unit_owner(rb * upr + upr - 1, U, g)
            if last > first:
                slots = max(slots, last - first + 1)
        jobs.append(dict(rbs=rbs, upr=upr, U=U, grid=g, rot=before % G, wait_for=wait_for,
                         slots=slots, part_off=part_off))
        before += U
        part_off += rbs * slots
    return jobs, part_off


def _segments(J, cta, G):
    c = cta + J["rot"]
    c -= G if c >= G else 0
    if c >= J["grid"]:
        return c, []
    ub, ue = _unit_begin(c, J["U"], J["grid"]), _unit_begin(c + 1, J["U"], J["grid"])
    segs, u = [], ub
    while u < ue:
        rb = u // J["upr"]
        end = min(ue, (rb + 1) * J["upr"])
        segs.append((rb, frozenset(range(u, end))))
        u = end
    return c, segs


def _share(J, cj, rb):
    first = _unit_owner(rb * J["upr"], J["U"], J["grid"])
    last = _unit_owner(rb * J["upr"] + J["upr"] - 1, J["U"], J["grid"])
    return last - first + 1, cj - first


def simulate(shapes, G, tags, seed, mistake=None):
    rnd = random.Random(seed)
    jobs, n_entries = _plan(shapes, G)
    ws = [0] * n_entries                     # zero-filled as handed over
    counts = [0] * (len(jobs) + 1)           # per job, then the exit counter
    for launch, tag in enumerate(tags):
        y = {}

        def cta(i):
            for j, J in enumerate(jobs):
                cj, segs = _segments(J, i, G)
                for rb, units in segs:
                    w = J["wait_for"]
                    if w >= 0:                # the activations wait for job w
                        while counts[w] < jobs[w]["rbs"]:
                            yield
                        assert all(y.get((w, r), (None,))[0] == launch
                                   for r in range(jobs[w]["rbs"])), "input read before written"
                    yield
                    value = (launch, units)
                    n, my = _share(J, cj, rb)
                    if n == 1:
                        if mistake == "count_before_write":
                            counts[j] += 1
                            yield
                            y[(j, rb)] = value
                        else:
                            y[(j, rb)] = value
                            counts[j] += 1
                        continue
                    base = J["part_off"] + rb * J["slots"]
                    if my != 0:
                        ws[base + my] = (0 if mistake == "untagged" else tag, value)
                        continue
                    got = [value]
                    for sl in range(1, n):
                        while mistake != "no_tag_wait" and not (ws[base + sl] != 0 and
                                                                ws[base + sl][0] == tag):
                            yield
                        entry = ws[base + sl]
                        got.append(entry[1] if entry != 0 else (None, frozenset()))
                    if mistake != "no_clear":
                        for sl in range(1, n):
                            ws[base + sl] = 0
                    launches = {g[0] for g in got}
                    assert launches == {launch}, "read another launch's partial sums"
                    if mistake == "count_before_write":
                        counts[j] += 1
                        yield
                    y[(j, rb)] = (launch, frozenset().union(*(g[1] for g in got)))
                    if mistake != "count_before_write":
                        counts[j] += 1
                    yield
            counts[-1] += 1
            if counts[-1] == G and mistake != "no_counter_reset":
                for k in range(len(counts)):
                    counts[k] = 0

        actors = {i: cta(i) for i in range(G)}
        speed = {i: rnd.choice([0.05, 1.0, 1.0, 4.0]) for i in actors}
        steps = 0
        while actors:
            steps += 1
            assert steps < 200000, "no progress"
            c = rnd.choices(list(actors), weights=[speed[a] for a in actors])[0]
            try:
                next(actors[c])
            except StopIteration:
                del actors[c]
        for j, J in enumerate(jobs):
            for rb in range(J["rbs"]):
                want = frozenset(range(rb * J["upr"], (rb + 1) * J["upr"]))
                assert y[(j, rb)] == (launch, want), (j, rb)
        assert all(e == 0 for e in ws), "workspace not left zero"
        assert all(c == 0 for c in counts), "counters not left zero"


# (row blocks, units per row block, wait_for) per job; CTA counts around the
# units of a job, so that row blocks are covered by one, two or many CTAs
SHAPES = [
    [(4, 10, -1)],
    [(48, 10, -1), (40, 34, 0), (136, 10, 1), (40, 34, 2)],
    [(3, 3, -1), (1, 7, 0), (5, 2, 1), (2, 9, 0)],
    [(1, 1, -1), (1, 30, 0), (30, 1, 1)],
]


@pytest.mark.parametrize("shapes", SHAPES)
@pytest.mark.parametrize("G", [1, 3, 7, 16])
def test_gemv_exchange_protocol(shapes, G):
    for seed in range(6):
        simulate(shapes, G, tags=[5, 5, 6], seed=seed)


@pytest.mark.parametrize("mistake", ["no_clear", "no_counter_reset", "untagged", "no_tag_wait",
                                     "count_before_write"])
def test_planted_mistakes_fail(mistake):
    for seed in range(30):
        try:
            simulate(SHAPES[2], 3 + seed % 5, tags=[5, 5, 6], seed=seed, mistake=mistake)
        except AssertionError:
            return
    raise AssertionError(f"the model did not catch {mistake}")
