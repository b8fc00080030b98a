"""The mbarrier protocol of the persistent tcgen05 attention kernel
(csrc/attend_tc.cuh), simulated on the host: no GPU.

Every role of one CTA is a coroutine that follows the kernel's order of
waits and arrivals over its work units: the two producer warps (each owning
alternate ring slots; producer 0 also loads q into one of two buffers), the
MMA thread (S(t) before P V(t - 1); the last P V of a unit commits o_full),
the four softmax warps (S read, P written, a rescale waiting for the
previous P V, (m_ref, l) left for the epilogue) and the four epilogue
warps.  Asynchronous completions (TMA bytes, tcgen05.commit arrivals) are
queued and delivered in random order.  A barrier keeps only the parity of
its phase, as the hardware does, so the simulation checks two things for
random unit and tile counts and ring depths:

- no role waits forever (every wait is eventually satisfied);
- no wait is satisfied by the wrong phase: a waiter is never two phases
  ahead of the barrier (the parity test would pass at once) nor behind it
  (the parity it waits for would come back only one phase later);
- no buffer is overwritten while it is still read: a unit's first P V into
  an O buffer, and the softmax's (m_ref, l) for a unit, come only after the
  epilogue warps have read that buffer's previous unit.

Mutants with one wait removed or one phase index off by one must fail, so
the checks are not vacuous."""
import random

import pytest


class _Barrier:
    def __init__(self, count):
        self.count, self.arrived, self.phase = count, 0, 0

    def arrive(self):
        self.arrived += 1
        assert self.arrived <= self.count
        if self.arrived == self.count:
            self.arrived, self.phase = 0, self.phase + 1


class ProtocolError(Exception):
    pass


def simulate(tiles_per_unit, stages=5, seed=0, mutant=None):
    """Run one CTA's roles over units with the given tile counts (0 = a unit
    without work, which every role skips).  Raises ProtocolError on a
    deadlock or a wait satisfied by the wrong phase."""
    rnd = random.Random(seed)
    bars = {}

    def bar(name, count):
        bars[name] = _Barrier(count)

    for s in range(stages):
        bar(f"full{s}", 1)
        bar(f"empty{s}", 1)
    for b in range(2):
        bar(f"s_full{b}", 1)
        bar(f"s_free{b}", 4)
        bar(f"p_full{b}", 4)
        bar(f"pv_done{b}", 1)
        bar(f"q_full{b}", 1)
        bar(f"q_empty{b}", 1)
        bar(f"o_full{b}", 1)
        bar(f"o_free{b}", 4)
        bar(f"ml_full{b}", 4)
    pending = []  # asynchronous arrivals, delivered in random order
    o_read = [dict(), dict()]  # O buffer -> {unit: epilogue warps done reading it}

    def check_o_free(k, who):
        ob = k & 1
        if k >= 2 and o_read[ob].get(k - 2, 0) != 4:
            raise ProtocolError(f"{who}: O buffer {ob} of unit {k - 2} overwritten while still read")

    def later(name):
        pending.append(name)

    def wait(name, index):
        return (name, index)

    work = [n for n in tiles_per_unit if n > 0]

    def producer(pidx):
        T = 0
        for k, n in enumerate(work):
            qb = k & 1
            if pidx == 0:
                if k >= 2:
                    yield wait(f"q_empty{qb}", (k >> 1) - 1 + (1 if mutant == "q_empty_index" else 0))
                later(f"q_full{qb}")
            for _ in range(n):
                slot = T % stages
                if (slot & 1) == pidx:
                    if T >= stages and mutant != "no_empty_wait":
                        yield wait(f"empty{slot}", T // stages - 1)
                    later(f"full{slot}")
                T += 1

    def mma():
        def pv(t, first, last, k):
            ob = k & 1
            yield wait(f"p_full{t & 1}", t >> 1)
            if first and k >= 2 and mutant != "no_o_free_wait":
                yield wait(f"o_free{ob}", (k >> 1) - 1)
            check_o_free(k, "mma")
            later(f"pv_done{t & 1}")
            later(f"empty{t % stages}")
            if last:
                later(f"o_full{ob}")

        prev, T = None, 0
        for k, n in enumerate(work):
            qb = k & 1
            yield wait(f"q_full{qb}", k >> 1)
            for t in range(n):
                yield wait(f"full{T % stages}", T // stages)
                if T >= 2:
                    yield wait(f"s_free{T & 1}", (T >> 1) - 1)
                later(f"s_full{T & 1}")
                if t == n - 1:
                    later(f"q_empty{qb}")
                if prev:
                    yield from pv(*prev)
                prev = (T, t == 0, t == n - 1, k)
                T += 1
        if prev:
            yield from pv(*prev)

    def softmax(warp):
        T = 0
        for k, n in enumerate(work):
            for t in range(n):
                yield wait(f"s_full{T & 1}", T >> 1)
                bars[f"s_free{T & 1}"].arrive()
                if T >= 2:
                    yield wait(f"pv_done{T & 1}", (T >> 1) - 1)
                if t >= 1 and rnd.random() < 0.3:  # a rescale of O: the previous P V first
                    yield wait(f"pv_done{(T - 1) & 1}", (T - 1) >> 1)
                bars[f"p_full{T & 1}"].arrive()
                T += 1
            ob = k & 1
            if k >= 2 and mutant != "no_ml_slot_wait":
                yield wait(f"o_free{ob}", (k >> 1) - 1)
            check_o_free(k, f"softmax{warp}")
            bars[f"ml_full{ob}"].arrive()

    def epilogue(warp):
        for k, _ in enumerate(work):
            ob = k & 1
            yield wait(f"o_full{ob}", k >> 1)
            yield wait(f"ml_full{ob}", k >> 1)
            yield None  # reads its O rows and (m_ref, l): other roles may run meanwhile
            o_read[ob][k] = o_read[ob].get(k, 0) + 1
            bars[f"o_free{ob}"].arrive()

    roles = {"producer0": producer(0), "producer1": producer(1), "mma": mma()}
    for w in range(4):
        roles[f"softmax{w}"] = softmax(w)
        roles[f"epilogue{w}"] = epilogue(w)
    waiting = {name: None for name in roles}
    done = set()
    while len(done) < len(roles):
        progressed = False
        order = list(roles)
        rnd.shuffle(order)
        for name in order:
            if name in done:
                continue
            if waiting[name] is not None:
                bname, index = waiting[name]
                b = bars[bname]
                # the hardware test: the phase of index's parity has completed
                # when the current phase (b.phase) has the other parity; right
                # only if the latest completed phase (b.phase - 1) is index
                if (b.phase & 1) != (index & 1):
                    if b.phase - 1 != index:
                        raise ProtocolError(f"{name}: {bname} phase {index} passes at {b.phase - 1} completed")
                    waiting[name] = None
                else:
                    if b.phase != index:
                        raise ProtocolError(f"{name}: {bname} phase {index} waited for at {b.phase - 1} completed")
                    continue
            try:
                waiting[name] = next(roles[name])  # None: a step that waits for nothing
            except StopIteration:
                done.add(name)
            progressed = True
        if pending and (not progressed or rnd.random() < 0.3):
            name = pending[rnd.randrange(len(pending))]
            bars[pending.pop(pending.index(name))].arrive()  # the oldest of that name: per-barrier order
            progressed = True
        if not progressed and not pending:
            raise ProtocolError(f"deadlock: {[(n, w) for n, w in waiting.items() if n not in done]}")


def _random_cases(count, seed):
    rnd = random.Random(seed)
    for trial in range(count):
        units = [rnd.choice([0, 1, 1, 2, 2, 3, 4, 5, 10]) for _ in range(rnd.randint(1, 9))]
        yield units, rnd.choice([2, 3, 4, 5, 6, 7]), trial


def test_protocol_has_no_deadlock_and_no_wrong_phase():
    for units, stages, trial in _random_cases(3000, 1):
        simulate(units, stages=stages, seed=trial)
    simulate([10] * 8, stages=5, seed=7)  # the ring depth the kernel uses, long units


@pytest.mark.parametrize("mutant", ["no_empty_wait", "q_empty_index", "no_o_free_wait", "no_ml_slot_wait"])
def test_protocol_mutants_are_caught(mutant):
    """One wait removed, or one waited-for phase off by one: some random case
    must deadlock or be satisfied by the wrong phase (or overfill a
    barrier's phase)."""
    caught = False
    for units, stages, trial in _random_cases(3000, 2):
        try:
            simulate(units, stages=stages, seed=trial, mutant=mutant)
        except (ProtocolError, AssertionError):
            caught = True
            break
    assert caught, mutant
