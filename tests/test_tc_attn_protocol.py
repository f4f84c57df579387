"""Host model of the synchronisation in the tensor-memory attention kernel
(q4kv_attn_tc.cuh): a producer thread (bulk copies into an S-slot ring), an
MMA thread, four K warps, four V warps and four softmax warps (one or two
P^T buffers; O^T rescaled only in tiles where a row maximum grows), coupled by
mbarriers that are waited on by phase parity.  Random interleavings
(asynchronous completions included) must always finish, every parity wait
must start while its barrier is at the awaited phase or one past it (else the
parity test passes early or never), and no buffer may be overwritten while an
asynchronous reader or writer still owns it."""
import random

import pytest

ROLE = 4   # warps per role


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.arrived, self.phase = name, count, 0, 0

    def arrive(self):
        self.arrived += 1
        assert self.arrived <= self.count, self.name
        if self.arrived == self.count:
            self.arrived = 0
            self.phase += 1


def simulate(n_tiles, S, seed, PB=2):
    rnd = random.Random(seed)
    full = [Bar(f"full{s}", 1) for s in range(S)]
    empty = [Bar(f"empty{s}", 2 * ROLE) for s in range(S)]
    kready = [Bar(f"kready{b}", ROLE) for b in range(2)]
    sdone = [Bar(f"sdone{b}", 1) for b in range(2)]
    pready = [Bar(f"pready{b}", ROLE) for b in range(PB)]
    pfree = [Bar(f"pfree{b}", 1) for b in range(PB)]
    vready = [Bar(f"vready{h}", ROLE) for h in range(2)]
    pvdone = [Bar(f"pvdone{h}", 1) for h in range(2)]
    pending_copies = []      # complete in any order
    pending_mma = []         # complete in issue order
    done = set()             # completed tensor-core work: ("qk", t), ("pv", h, t)
    state = {"ring": [None] * S, "released": {}, "s_read": {}, "k_written": {},
             "p_written": set(), "v_written": set(), "rescale": {}}

    def wait(bar, k):
        # parity wait for phase k: phases < k complete, phase k + 1 not yet
        assert k <= bar.phase <= k + 1, (bar.name, k, bar.phase)
        while bar.phase <= k:
            yield

    def producer():
        for t in range(n_tiles):
            slot = t % S
            if t >= S:
                yield from wait(empty[slot], t // S - 1)
                assert state["released"].get(t - S, 0) == 2 * ROLE
            state["ring"][slot] = t
            pending_copies.append(slot)
            yield

    def mma():
        def qk(t):
            b = t & 1
            yield from wait(kready[b], t >> 1)
            if t >= 2:
                # S^T[b] free: PV(t - 2), issued before, waited for the softmax of t - 2
                assert state["s_read"].get(t - 2, 0) == ROLE
            assert state["k_written"].get(t, 0) == ROLE
            pending_mma.append(("qk", t))
            yield

        if n_tiles:
            yield from qk(0)
        for t in range(n_tiles):
            if t + 1 < n_tiles:
                yield from qk(t + 1)
            yield from wait(pready[t % PB], t // PB)
            for h in range(2):
                yield from wait(vready[h], t)
                assert (t, h) in state["v_written"] and t in state["p_written"]
                pending_mma.append(("pv", h, t))
                yield
            pending_mma.append(("pfree", t))

    def k_warp(w):
        for t in range(n_tiles):
            slot = t % S
            yield from wait(full[slot], t // S)
            assert state["ring"][slot] == t
            if t >= 2:
                yield from wait(sdone[t & 1], (t - 2) >> 1)
                assert ("qk", t - 2) in done                   # K buffer free
            state["k_written"][t] = state["k_written"].get(t, 0) + 1
            kready[t & 1].arrive()
            state["released"][t] = state["released"].get(t, 0) + 1
            empty[slot].arrive()
            yield

    def v_warp(w):
        for t in range(n_tiles):
            slot = t % S
            yield from wait(full[slot], t // S)
            assert state["ring"][slot] == t
            for h in range(2):
                if t > 0:
                    yield from wait(pvdone[h], t - 1)
                    assert ("pv", h, t - 1) in done            # V half free
                state["v_written"].add((t, h))
                vready[h].arrive()
                yield
            assert state["ring"][slot] == t
            state["released"][t] = state["released"].get(t, 0) + 1
            empty[slot].arrive()

    def softmax_warp(w):
        for t in range(n_tiles):
            yield from wait(sdone[t & 1], t >> 1)
            assert ("qk", t) in done
            state["s_read"][t] = state["s_read"].get(t, 0) + 1
            yield "barrier"
            # the CTA-wide rescale decision of tile t (same for every warp)
            rescale = state["rescale"].setdefault(t, rnd.random() < 0.3)
            yield "barrier"
            if t >= PB:
                yield from wait(pfree[t % PB], (t - PB) // PB)
                assert ("pv", 1, t - PB) in done               # P^T buffer free
            if rescale and t > 0:
                yield from wait(pvdone[1], t - 1)
                assert ("pv", 0, t - 1) in done and ("pv", 1, t - 1) in done   # O^T idle
            state["p_written"].add(t)
            pready[t % PB].arrive()
            yield
        if n_tiles:
            yield from wait(pfree[(n_tiles - 1) % PB], (n_tiles - 1) // PB)
            assert all(("pv", h, n_tiles - 1) in done for h in range(2))

    actors = {"producer": producer(), "mma": mma()}
    for w in range(ROLE):
        actors[("k", w)] = k_warp(w)
        actors[("v", w)] = v_warp(w)
        actors[("s", w)] = softmax_warp(w)
    # per-run random speeds, so that some schedules starve one actor
    speed = {a: rnd.choice([0.05, 1.0, 1.0, 4.0]) for a in actors}
    speed["copy"], speed["tensor"] = rnd.choice([0.1, 1.0, 4.0]), rnd.choice([0.1, 1.0, 4.0])
    at_barrier = set()
    steps = 0
    while actors or pending_copies or pending_mma:
        steps += 1
        assert steps < 400000, "no progress"
        choices = [a for a in actors if a not in at_barrier]
        choices += ["copy"] * bool(pending_copies) + ["tensor"] * bool(pending_mma)
        assert choices, f"deadlock: {sorted(map(str, actors))}"
        c = rnd.choices(choices, weights=[speed[x] for x in choices])[0]
        if c == "copy":
            full[pending_copies.pop(rnd.randrange(len(pending_copies)))].arrive()
            continue
        if c == "tensor":
            job = pending_mma.pop(0)
            done.add(job)
            if job[0] == "qk":
                sdone[job[1] & 1].arrive()
            elif job[0] == "pv":
                pvdone[job[1]].arrive()
            else:
                pfree[job[1] % PB].arrive()
            continue
        try:
            if next(actors[c]) == "barrier":
                at_barrier.add(c)
                if all(a in at_barrier for a in actors if isinstance(a, tuple) and a[0] == "s"):
                    at_barrier.clear()
        except StopIteration:
            del actors[c]
    assert all(("pv", h, t) in done for t in range(n_tiles) for h in range(2))
    assert all(("pfree", t) in done for t in range(n_tiles))


@pytest.mark.parametrize("n_tiles,S", [(1, 2), (2, 2), (3, 2), (3, 3), (5, 3), (9, 4), (16, 3), (4, 8)])
@pytest.mark.parametrize("PB", [1, 2])
def test_tc_attention_protocol(n_tiles, S, PB):
    for seed in range(60):
        simulate(n_tiles, S, seed, PB)
