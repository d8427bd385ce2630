"""A model of the tensor-core output pass's mbarrier protocol, run on the CPU.

The output pass (single CTA, and the CTA pair) is a pipeline of roles that
meet only on mbarriers: a producer issuing TMA loads into a ring of slots,
an MMA thread, mask/epilogue warpgroups and, in the pair's fold mode, fold
warps.  A barrier phase is observed through its parity, so a waiter that
runs two phases ahead of a barrier sees an older phase's completion as the
one it wants.  This model replays the roles' barrier operations in the
order the kernels issue them (ring items per work item: the query tile, the
key tiles, the state halves, the value tiles, the gate/output tile), under
random interleavings and random arrival times of the loads, and checks that
every run finishes without a deadlock or an over-arrival.  The single CTA's
MMA waits also state the number of completions they need, so a wait that
passes on an older phase of the same parity is reported when it happens.

It also keeps, as `aliasing=True`, the protocol the kernels had before: the
gate tile counted on its slot's full barrier (single CTA) and raw q counted
on its slot's local barrier (pair, fold mode).  The model must find those
races, so that it is known to be able to find one.
"""
import random

import pytest


class Barrier:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.tx, self.phase = name, count, count, 0, 0

    def arrive(self):
        self.pending -= 1
        self._settle()

    def expect_tx(self, n):
        self.tx += n
        self.arrive()

    def land(self, n):
        self.tx -= n
        self._settle()

    def _settle(self):
        if self.pending < 0:
            raise OverArrival(self.name)
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def passed(self, parity):                   # mbarrier.try_wait.parity
        return (self.phase & 1) != parity


class OverArrival(Exception):
    pass


class StaleWait(Exception):
    """A wait given the number of completions it needs passed before them."""


def simulate(roles, inflight, rng, limit=400000):
    """Run generator roles that yield (barrier, parity) waits, or (barrier,
    parity, completions needed) to have a stale pass reported; None on
    success, else a description of the deadlock."""
    waiting = [None] * len(roles)
    alive = list(range(len(roles)))
    for _ in range(limit):
        if not alive:
            return None
        progressed = False
        rng.shuffle(inflight)
        k = rng.randint(0, len(inflight))
        for bar, n in inflight[:k]:
            bar.land(n)
        del inflight[:k]
        order = alive[:]
        rng.shuffle(order)
        for i in order:
            if waiting[i] is not None:
                bar, par = waiting[i][0], waiting[i][1]
                if not bar.passed(par):
                    continue
                if len(waiting[i]) > 2 and bar.phase < waiting[i][2]:
                    raise StaleWait(bar.name)   # passed on an older phase of the same parity
                waiting[i] = None
            try:
                waiting[i] = next(roles[i])
                progressed = True
            except StopIteration:
                alive.remove(i)
                progressed = True
        if not progressed and not inflight:
            return [(waiting[i][0].name, waiting[i][1]) for i in alive if waiting[i]]
    return "no end"


def ring_items(nk, nsp):
    """Ring order of one work item: query, key(0), then per key tile t:
    key(t+1), state half t (t < nsp), value(t); the rest of the state halves;
    the gate/output tile.  Returns kinds."""
    kinds = ["q", "k"]
    for t in range(nk):
        if t + 1 < nk:
            kinds.append("k")
        if t < nsp:
            kinds.append("s")
        kinds.append("v")
    kinds += ["s"] * max(0, nsp - nk)
    kinds.append("g")
    return kinds


# ------------------------------------------------------------------ single CTA
def single_cta(items, gate, aliasing, rng, slots=3):
    B = {}
    for s in range(slots):
        B[f"full{s}"] = Barrier(f"full{s}", 1)
        B[f"empty{s}"] = Barrier(f"empty{s}", 1)
    for name, count in (("s_full", 1), ("s_read", 2), ("p_full0", 1), ("p_full1", 1),
                        ("p_free0", 1), ("p_free1", 1), ("o_full", 1), ("o_free", 2),
                        ("g_full", 1), ("epi", 2)):
        B[name] = Barrier(name, count)
    inflight = []

    def producer():
        it = 0
        for nk, nsp in items:
            for kind in ring_items(nk, nsp):
                s = it % slots
                if it >= slots:
                    yield B[f"empty{s}"], ((it // slots) - 1) & 1
                if kind == "g" and not aliasing:
                    if gate:
                        B["g_full"].expect_tx(1)
                        inflight.append((B["g_full"], 1))
                    else:
                        B["g_full"].arrive()
                elif kind == "g" and not gate:
                    B[f"full{s}"].arrive()
                else:
                    B[f"full{s}"].expect_tx(1)
                    inflight.append((B[f"full{s}"], 1))
                it += 1

    def mma():
        it = nqk = npv = 0
        par = [0] * slots
        ops = [0] * slots                       # operand phases of each slot taken so far

        def take():
            s = it % slots
            if aliasing:                        # every ring item is a phase of its slot
                yield B[f"full{s}"], (it // slots) & 1, it // slots + 1
            else:                               # only the slot's operand tiles are
                yield B[f"full{s}"], par[s], ops[s] + 1
                par[s] ^= 1
                ops[s] += 1

        for li, (nk, nsp) in enumerate(items):
            written = [False]

            def claim():
                if not written[0] and li > 0:
                    yield B["o_free"], (li - 1) & 1
                written[0] = True

            if li > 0:
                yield B["o_full"], (li - 1) & 1      # the query copy waits for the last MMAs
            yield from take()
            B[f"empty{it % slots}"].arrive()
            it += 1

            def qk():
                nonlocal it, nqk
                if nqk:
                    yield B["s_read"], (nqk - 1) & 1
                yield from take()
                B[f"empty{it % slots}"].arrive()
                B["s_full"].arrive()
                it += 1
                nqk += 1

            def qs():
                nonlocal it
                yield from take()
                yield from claim()
                B[f"empty{it % slots}"].arrive()
                it += 1

            yield from qk()
            for t in range(nk):
                if t + 1 < nk:
                    yield from qk()
                if t < nsp:
                    yield from qs()
                yield from take()
                yield from claim()
                for hx in range(2):
                    yield B[f"p_full{hx}"], npv & 1
                    B[f"p_free{hx}"].arrive()
                B[f"empty{it % slots}"].arrive()
                it += 1
                npv += 1
            for _ in range(nk, nsp):
                yield from qs()
            B["o_full"].arrive()
            it += 1

    def warpgroup(wg):
        base = ntile = 0
        for li, (nk, nsp) in enumerate(items):
            for _ in range(nk):
                yield B["s_full"], ntile & 1
                B["s_read"].arrive()
                if ntile:
                    yield B[f"p_free{wg}"], (ntile - 1) & 1
                B[f"p_full{wg}"].arrive()
                ntile += 1
            ig = base + len(ring_items(nk, nsp)) - 1
            base = ig + 1
            yield B["o_full"], li & 1
            if aliasing:
                yield B[f"full{ig % slots}"], (ig // slots) & 1
            else:
                yield B["g_full"], li & 1
            B["o_free"].arrive()
            B["epi"].arrive()                       # the warpgroups' named barrier
            yield B["epi"], li & 1
            if wg == 0:
                B[f"empty{ig % slots}"].arrive()

    return simulate([producer(), mma(), warpgroup(0), warpgroup(1)], inflight, rng)


# ------------------------------------------------------------------ CTA pair
def cta_pair(items, gate, fold, aliasing, rng, slots=6):
    B = {}

    def bar(name, count):
        B[name] = Barrier(name, count)

    for c in (0, 1):
        for s in range(slots):
            bar(f"full{s}.{c}", 1)
            bar(f"empty{s}.{c}", 1)
            bar(f"local{s}.{c}", 1)
        for name, count in (("s_full", 1), ("s_read", 4), ("p_full0", 2), ("p_full1", 2),
                            ("p_free0", 1), ("p_free1", 1), ("o_full", 1), ("o_free", 4),
                            ("q_ready", 2), ("qfull0", 1), ("qfull1", 1), ("epi", 2)):
            bar(f"{name}.{c}", count)
    inflight = []

    def producer(c):
        it = 0
        for nk, nsp in items:
            kinds = ring_items(nk, nsp)
            kinds = [kinds[0], "q"] + kinds[1:-1] + ["g", "g"]     # two query and gate halves
            half = 0
            for kind in kinds:
                s = it % slots
                if it >= slots:
                    yield B[f"empty{s}.{c}"], ((it // slots) - 1) & 1
                local = B[f"local{s}.{c}"]
                if kind == "q" and fold:
                    if aliasing:
                        local.expect_tx(1)
                        inflight.append((local, 1))
                    else:
                        local.arrive()
                        q = B[f"qfull{half}.{c}"]
                        q.expect_tx(1)
                        inflight.append((q, 1))
                    half ^= 1
                elif kind == "g":
                    if gate:
                        local.expect_tx(1)
                        inflight.append((local, 1))
                    else:
                        local.arrive()
                else:
                    local.arrive()
                    if c == 0:
                        B[f"full{s}.0"].expect_tx(2)
                    inflight.append((B[f"full{s}.0"], 1))
                it += 1

    def mma():
        it = nqk = npv = 0
        par = [0] * slots

        def commit(name):
            for c in (0, 1):
                B[f"{name}.{c}"].arrive()

        def take():
            s = it % slots
            yield B[f"full{s}.0"], par[s]
            par[s] ^= 1

        for li, (nk, nsp) in enumerate(items):
            written = [False]

            def claim():
                if not written[0] and li > 0:
                    yield B["o_free.0"], (li - 1) & 1
                written[0] = True

            if li > 0:
                yield B["o_full.0"], (li - 1) & 1
            if fold:
                yield B["q_ready.0"], li & 1
            else:
                yield from take()
            sa = it % slots
            it += 1
            if not fold:
                yield from take()
            sb = it % slots
            it += 1
            commit(f"empty{sa}")
            commit(f"empty{sb}")

            def qk():
                nonlocal it, nqk
                if nqk:
                    yield B["s_read.0"], (nqk - 1) & 1
                yield from take()
                commit(f"empty{it % slots}")
                commit("s_full")
                it += 1
                nqk += 1

            def qs():
                nonlocal it
                yield from take()
                yield from claim()
                commit(f"empty{it % slots}")
                it += 1

            yield from qk()
            for t in range(nk):
                if t + 1 < nk:
                    yield from qk()
                if t < nsp:
                    yield from qs()
                yield from take()
                yield from claim()
                for hx in range(2):
                    yield B[f"p_full{hx}.0"], npv & 1
                    commit(f"p_free{hx}")
                commit(f"empty{it % slots}")
                it += 1
                npv += 1
            for _ in range(nk, nsp):
                yield from qs()
            commit("o_full")
            it += 2

    def folder(c):
        base = 0
        for li, (nk, nsp) in enumerate(items):
            for half in range(2):
                if aliasing:
                    qs = base + half
                    yield B[f"local{qs % slots}.{c}"], (qs // slots) & 1
                else:
                    yield B[f"qfull{half}.{c}"], li & 1
            B["q_ready.0"].arrive()
            base += len(ring_items(nk, nsp)) + 2

    def warpgroup(c, wg):
        base = ntile = 0
        for li, (nk, nsp) in enumerate(items):
            for _ in range(nk):
                yield B[f"s_full.{c}"], ntile & 1
                B["s_read.0"].arrive()
                if ntile:
                    yield B[f"p_free{wg}.{c}"], (ntile - 1) & 1
                B[f"p_full{wg}.0"].arrive()
                ntile += 1
            ig = base + len(ring_items(nk, nsp))     # the first of the two gate slots
            base = ig + 2
            yield B[f"o_full.{c}"], li & 1
            for j in (ig, ig + 1):
                yield B[f"local{j % slots}.{c}"], (j // slots) & 1
            B["o_free.0"].arrive()
            B[f"epi.{c}"].arrive()
            yield B[f"epi.{c}"], li & 1
            if wg == 0:
                B[f"empty{ig % slots}.{c}"].arrive()
                B[f"empty{(ig + 1) % slots}.{c}"].arrive()

    roles = [producer(0), producer(1), mma()] + [warpgroup(c, wg) for c in (0, 1) for wg in (0, 1)]
    if fold:
        roles += [folder(0), folder(1)]
    return simulate(roles, inflight, rng)


def random_items(rng, short):
    n = rng.randint(1, 12)
    if short:                                   # chunk 128: one key tile per item
        return [(1, rng.choice([0, 2])) for _ in range(n)]
    return [(rng.randint(1, 6), rng.choice([0, 2])) for _ in range(n)]


def failures(run, seeds, **kw):
    bad = 0
    for seed in range(seeds):
        rng = random.Random(seed)
        items = random_items(rng, short=seed % 2 == 0)
        try:
            result = run(items, rng=rng, **kw)
        except OverArrival:
            result = "over-arrival"
        except StaleWait:
            result = "stale wait"
        bad += result is not None
    return bad


@pytest.mark.parametrize("gate", [True, False])
def test_single_cta_protocol_has_no_race(gate):
    assert failures(single_cta, 400, gate=gate, aliasing=False) == 0


def test_single_cta_model_finds_the_gate_aliasing_race():
    assert failures(single_cta, 3000, gate=True, aliasing=True) > 0


@pytest.mark.parametrize("fold", [True, False])
@pytest.mark.parametrize("gate", [True, False])
def test_cta_pair_protocol_has_no_race(fold, gate):
    assert failures(cta_pair, 150, gate=gate, fold=fold, aliasing=False) == 0


def test_cta_pair_model_finds_the_fold_aliasing_race():
    assert failures(cta_pair, 150, gate=True, fold=True, aliasing=True) > 0

